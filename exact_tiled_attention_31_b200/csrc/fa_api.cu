// fa_api.cu - host side of the C ABI declared in include/fa.h: argument
// checks, TMA tensor-map encoding, launch configuration and the device error
// word.  All device work happens in the kernels of fa_fwd.cuh / fa_bwd.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <initializer_list>
#include <mutex>
#include <utility>

#include "../../include/fa.h"
#include "fa_bwd.cuh"
#include "fa_decode.cuh"
#include "fa_fwd.cuh"

namespace {

std::atomic<uint64_t> g_launches{0};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// [heads, rows, D] 16-bit tensor, boxes of box_rows rows x 64 columns, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int D, long long rows, long long heads, bool bf16,
              unsigned box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)heads};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
             const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 dQ accumulator [heads, rows, D] for TMA bulk reductions: boxes of
// 32 rows x 32 columns (128 bytes), 128-byte swizzle.
bool make_map_f32(CUtensorMap* m, const void* base, int D, long long rows, long long heads) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)heads};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)rows * D * 4};
  const cuuint32_t box[3] = {32, 32, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Per-query rows of the backward's extra K step: bf16 [rows, 16], boxes of
// 128 rows x 16 columns (32 bytes), 32-byte swizzle.
bool make_map_cols(CUtensorMap* m, const void* base, long long rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {16, (cuuint64_t)rows, 1};
  const cuuint64_t strides[2] = {32, (cuuint64_t)rows * 32};
  const cuuint32_t box[3] = {16, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool scale_ok(float s) { return std::isfinite(s) && s > 0.f; }

// Opt every kernel instance into its dynamic shared memory once per device
// (one flag word per instance: the template argument is the kernel itself).
template <auto Kernel>
cudaError_t set_smem(uint32_t bytes) {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load() & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) done.fetch_or(bit);
  return e;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

fa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? FA_OK : FA_ERR_CUDA; }

// ---------------------------------------------------------------- forward
template <int D, bool BF16, bool CAUSAL, bool VARLEN, bool DROPOUT = false>
fa_status launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const fa::FwdParams& p,
                     cudaStream_t st) {
  using C = fa::FwdCfg<D>;
  auto kern = fa::fwd_kernel<D, BF16, CAUSAL, VARLEN, DROPOUT>;
  cudaError_t e = set_smem<fa::fwd_kernel<D, BF16, CAUSAL, VARLEN, DROPOUT>>(C::SMEM);
  if (e != cudaSuccess) return FA_ERR_CUDA;
  const long long grid = (long long)p.n_pairs * p.nseq * p.heads;
  if (grid <= 0) return FA_OK;
  if (grid > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  kern<<<(unsigned)grid, C::THREADS, C::SMEM, st>>>(mq, mk, mv, p);
  g_launches.fetch_add(1);
  return from_cuda(cudaGetLastError());
}

template <int D, bool BF16>
fa_status dispatch_fwd(bool causal, bool varlen, bool dropout, const CUtensorMap& mq, const CUtensorMap& mk,
                       const CUtensorMap& mv, const fa::FwdParams& p, cudaStream_t st) {
  if (dropout)
    return varlen ? (causal ? launch_fwd<D, BF16, true, true, true>(mq, mk, mv, p, st)
                            : launch_fwd<D, BF16, false, true, true>(mq, mk, mv, p, st))
                  : (causal ? launch_fwd<D, BF16, true, false, true>(mq, mk, mv, p, st)
                            : launch_fwd<D, BF16, false, false, true>(mq, mk, mv, p, st));
  if (varlen)
    return causal ? launch_fwd<D, BF16, true, true>(mq, mk, mv, p, st)
                  : launch_fwd<D, BF16, false, true>(mq, mk, mv, p, st);
  return causal ? launch_fwd<D, BF16, true, false>(mq, mk, mv, p, st)
                : launch_fwd<D, BF16, false, false>(mq, mk, mv, p, st);
}

fa_status run_fwd(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu, int heads,
                  int seqlen, long long rows, int nseq, int D, float scale, bool causal, bool bf16, bool varlen,
                  cudaStream_t st, const fa::Dropout* drop = nullptr) {
  // query and key/value tiles of 128 rows
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, D, rows, heads, bf16, 128) || !make_map(&mk, k, D, rows, heads, bf16, 128) ||
      !make_map(&mv, v, D, rows, heads, bf16, 128))
    return FA_ERR_CUDA;
  fa::FwdParams p;
  p.o = o;
  p.lse = lse;
  p.cu_seqlens = cu;
  p.heads = heads;
  p.seqlen = seqlen;
  p.rows = (int)rows;
  p.nseq = nseq;
  p.n_pairs = (seqlen + 255) / 256;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.drop = drop ? *drop : fa::Dropout{};
  const bool dr = drop != nullptr;
  if (D == 64)
    return bf16 ? dispatch_fwd<64, true>(causal, varlen, dr, mq, mk, mv, p, st)
                : dispatch_fwd<64, false>(causal, varlen, dr, mq, mk, mv, p, st);
  return bf16 ? dispatch_fwd<128, true>(causal, varlen, dr, mq, mk, mv, p, st)
              : dispatch_fwd<128, false>(causal, varlen, dr, mq, mk, mv, p, st);
}

// ---------------------------------------------------------------- backward
struct WsLayout {
  size_t dq_acc, cols, sem, ticket, total;
};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// heads x rows token rows in memory; per-query rows (16 bf16 each) padded per
// sequence to ceil(S / 128) * 128 rows (S = the longest sequence)
WsLayout ws_layout(long long heads, long long nseq, long long S, long long rows, int D) {
  const long long n_q = (S + 127) / 128, S_pad = n_q * 128;
  WsLayout w;
  w.dq_acc = 0;  // two fp32 accumulators back to back (the second for deterministic mode)
  w.cols = up256((size_t)2 * heads * rows * D * 4);
  w.sem = w.cols + up256((size_t)heads * nseq * S_pad * 32);
  w.ticket = w.sem + up256((size_t)heads * nseq * n_q * 2 * 4);
  w.total = w.ticket + 256;
  return w;
}

fa::BwdParams bwd_params(int heads, int nseq, int S, int rows, const int* cu, int D, float scale, int deterministic,
                         uint8_t* ws, void* dk, void* dv) {
  const WsLayout w = ws_layout(heads, nseq, S, rows, D);
  fa::BwdParams p;
  p.dk = dk;
  p.dv = dv;
  p.dq_acc = reinterpret_cast<float*>(ws + w.dq_acc);
  p.cols = reinterpret_cast<uint16_t*>(ws + w.cols);
  p.sem = reinterpret_cast<uint32_t*>(ws + w.sem);
  p.ticket = reinterpret_cast<uint32_t*>(ws + w.ticket);
  p.cu_seqlens = cu;
  p.heads = heads;
  p.S = S;
  p.rows = rows;
  p.nseq = nseq;
  p.n_q = (S + 127) / 128;
  p.S_pad = p.n_q * 128;
  const long long groups = ((long long)heads * nseq + fa::kBwdGroup - 1) / fa::kBwdGroup;
  const long long units = groups * fa::kBwdGroup * p.n_q;
  p.units = units > 0x7fffffffLL ? -1 : (int)units;  // -1: too many for one launch
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.deterministic = deterministic;
  p.drop = fa::Dropout{};
  return p;
}

template <int D, bool BF16>
fa_status launch_bwd_pre(const void* o, const void* dO, const float* lse, const fa::BwdParams& p, bool varlen,
                         cudaStream_t st) {
  const uint16_t* o16 = static_cast<const uint16_t*>(o);
  const uint16_t* do16 = static_cast<const uint16_t*>(dO);
  // y: (head, sequence) slices (looped past 65535); x: about eight blocks per
  // SM in all, at least one, at most enough for one pass over a slice's rows
  const long long slices = (long long)p.heads * p.nseq;
  if ((long long)p.S_pad * (D / 8) + 31 > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;  // 32-bit row indices
  const int gy = (int)std::min<long long>(slices, 65535);
  const long long per_slice = ((long long)p.S_pad * (D / 8) + 255) / 256;
  const int gx = (int)std::max<long long>(1, std::min<long long>(per_slice, (sm_count() * 8LL + gy - 1) / gy));
  const dim3 grid(gx, gy);
  if (varlen)
    fa::bwd_pre_kernel<D, BF16, true><<<grid, 256, 0, st>>>(o16, do16, lse, p);
  else
    fa::bwd_pre_kernel<D, BF16, false><<<grid, 256, 0, st>>>(o16, do16, lse, p);
  g_launches.fetch_add(1);
  return from_cuda(cudaGetLastError());
}

template <int D, bool BF16, bool CAUSAL, bool VARLEN, bool DROPOUT, bool DET>
fa_status launch_bwd_main_det(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                              const CUtensorMap& mdo, const CUtensorMap& mdq, const CUtensorMap& mcols,
                              const fa::BwdParams& p, cudaStream_t st) {
  using C = fa::BwdCfg<D>;
  const int grid = std::min(p.units, sm_count());
  if (set_smem<fa::bwd_main_kernel<D, BF16, CAUSAL, VARLEN, DROPOUT, DET>>(C::SMEM) != cudaSuccess)
    return FA_ERR_CUDA;
  fa::bwd_main_kernel<D, BF16, CAUSAL, VARLEN, DROPOUT, DET><<<(unsigned)grid, 512, C::SMEM, st>>>(
      mq, mk, mv, mdo, mdq, mcols, p);
  return FA_OK;
}

template <int D, bool BF16, bool CAUSAL, bool VARLEN, bool DROPOUT = false>
fa_status launch_bwd_main_t(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                            const CUtensorMap& mdo, const CUtensorMap& mdq, const CUtensorMap& mcols,
                            const fa::BwdParams& p, cudaStream_t st) {
  // persistent grid: at most one CTA per SM, each claiming units from the
  // workspace counter that bwd_pre zeroed
  if (p.units < 0) return FA_ERR_UNSUPPORTED;
  if (p.units == 0) return FA_OK;
  const fa_status s = p.deterministic
                          ? launch_bwd_main_det<D, BF16, CAUSAL, VARLEN, DROPOUT, true>(mq, mk, mv, mdo, mdq, mcols, p, st)
                          : launch_bwd_main_det<D, BF16, CAUSAL, VARLEN, DROPOUT, false>(mq, mk, mv, mdo, mdq, mcols, p, st);
  if (s != FA_OK) return s;
  g_launches.fetch_add(1);
  return from_cuda(cudaGetLastError());
}

template <int D, bool BF16>
fa_status launch_bwd_main(const void* q, const void* k, const void* v, const void* dO, const fa::BwdParams& p,
                          bool causal, bool varlen, bool dropout, cudaStream_t st) {
  if (p.deterministic) {
    // the second accumulator (odd key tiles) starts at zero, and the flag
    // tells bwd_post to add it
    const size_t n = (size_t)p.heads * p.rows * D;
    if (cudaMemsetAsync(p.dq_acc + n, 0, n * 4, st) != cudaSuccess ||
        cudaMemsetAsync(p.ticket + 1, 1, 1, st) != cudaSuccess)
      return FA_ERR_CUDA;
  }
  CUtensorMap mq, mk, mv, mdo, mdq, mcols;
  if (!make_map(&mq, q, D, p.rows, p.heads, BF16) || !make_map(&mk, k, D, p.rows, p.heads, BF16) ||
      !make_map(&mv, v, D, p.rows, p.heads, BF16) || !make_map(&mdo, dO, D, p.rows, p.heads, BF16) ||
      !make_map_f32(&mdq, p.dq_acc, D, p.rows, 2LL * p.heads) ||
      !make_map_cols(&mcols, p.cols, (long long)p.heads * p.nseq * p.S_pad))
    return FA_ERR_CUDA;
  if (dropout)
    return varlen ? (causal ? launch_bwd_main_t<D, BF16, true, true, true>(mq, mk, mv, mdo, mdq, mcols, p, st)
                            : launch_bwd_main_t<D, BF16, false, true, true>(mq, mk, mv, mdo, mdq, mcols, p, st))
                  : (causal ? launch_bwd_main_t<D, BF16, true, false, true>(mq, mk, mv, mdo, mdq, mcols, p, st)
                            : launch_bwd_main_t<D, BF16, false, false, true>(mq, mk, mv, mdo, mdq, mcols, p, st));
  if (varlen)
    return causal ? launch_bwd_main_t<D, BF16, true, true>(mq, mk, mv, mdo, mdq, mcols, p, st)
                  : launch_bwd_main_t<D, BF16, false, true>(mq, mk, mv, mdo, mdq, mcols, p, st);
  return causal ? launch_bwd_main_t<D, BF16, true, false>(mq, mk, mv, mdo, mdq, mcols, p, st)
                : launch_bwd_main_t<D, BF16, false, false>(mq, mk, mv, mdo, mdq, mcols, p, st);
}

// det: bwd_main ran deterministic (two accumulators to add)
template <bool BF16>
fa_status launch_bwd_post(void* dq, const fa::BwdParams& p, int D, cudaStream_t st, bool det) {
  const long long n8 = (long long)p.heads * p.rows * D / 8;
  // 8 CTAs of 256 threads per SM, all resident at once
  if (det)
    fa::bwd_post_kernel<BF16, true><<<sm_count() * 8, 256, 0, st>>>(p.dq_acc, p.ticket + 1,
                                                                     static_cast<uint16_t*>(dq), n8, p.scale);
  else
    fa::bwd_post_kernel<BF16, false><<<sm_count() * 8, 256, 0, st>>>(p.dq_acc, p.ticket + 1,
                                                                      static_cast<uint16_t*>(dq), n8, p.scale);
  g_launches.fetch_add(1);
  return from_cuda(cudaGetLastError());
}

// The three backward launches over prepared parameters (dense or packed).
fa_status run_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                  void* dq, const fa::BwdParams& p, int D, bool causal, bool bf16, bool varlen, cudaStream_t st,
                  bool dropout = false) {
  fa_status c;
  if (D == 64)
    c = bf16 ? launch_bwd_pre<64, true>(o, dO, lse, p, varlen, st) : launch_bwd_pre<64, false>(o, dO, lse, p, varlen, st);
  else
    c = bf16 ? launch_bwd_pre<128, true>(o, dO, lse, p, varlen, st)
             : launch_bwd_pre<128, false>(o, dO, lse, p, varlen, st);
  if (c != FA_OK) return c;
  if (D == 64)
    c = bf16 ? launch_bwd_main<64, true>(q, k, v, dO, p, causal, varlen, dropout, st)
             : launch_bwd_main<64, false>(q, k, v, dO, p, causal, varlen, dropout, st);
  else
    c = bf16 ? launch_bwd_main<128, true>(q, k, v, dO, p, causal, varlen, dropout, st)
             : launch_bwd_main<128, false>(q, k, v, dO, p, causal, varlen, dropout, st);
  if (c != FA_OK) return c;
  return bf16 ? launch_bwd_post<true>(dq, p, D, st, p.deterministic != 0)
              : launch_bwd_post<false>(dq, p, D, st, p.deterministic != 0);
}

// shared checks of the backward entry points: sizes, dtype, workspace
fa_status bwd_common_checks(int B, int H, int S, int D, fa_dtype dt, const void* workspace, size_t workspace_bytes) {
  if (B < 0 || H < 0 || S < 0) return FA_ERR_INVALID_ARG;
  if (dt != FA_BF16 && dt != FA_FP16) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if ((long long)B * H > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || S == 0) return FA_OK;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return FA_ERR_INVALID_ARG;
  size_t need = ws_layout((long long)B * H, 1, S, S, D).total;
  if (workspace_bytes < need) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

bool ptrs_ok(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (!p || !aligned16(p)) return false;
  return true;
}

// ---------------------------------------------------------------- error-path self-test
// One warp waits, through the same bounded wait every kernel uses, on an
// mbarrier that nothing ever arrives on: after the wait limit it records the
// timeout in the device error word and returns normally.
__global__ void __launch_bounds__(32) selftest_timeout_kernel() {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    fa::mbar_init(&bar, 1);
    fa::fence_mbar_init();
  }
  __syncwarp();
  fa::mbar_wait(&bar, 0, 0x300);
}

// ---------------------------------------------------------------- allocation-free backward
// Scratch of fa_bwd_noalloc: a fixed array in device memory, created when
// the library's module is loaded on a device and held until the process
// exits.  Host code only sees a host-side stand-in under this name; the
// device address is looked up once per device below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[FA_BWD_NOALLOC_SCRATCH_BYTES];

// Process-unique id of the calling thread's current CUDA context
// (cuCtxGetId), or 0 when the driver does not offer it.  Ids are never
// reused within a process, unlike context handles after a reset.
unsigned long long current_context_id() {
  using GetCurrentFn = CUresult (*)(CUcontext*);
  using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
  static const std::pair<GetCurrentFn, GetIdFn> fns = []() -> std::pair<GetCurrentFn, GetIdFn> {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) != cudaSuccess ||
        qa != cudaDriverEntryPointSuccess || cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) != cudaSuccess ||
        qb != cudaDriverEntryPointSuccess)
      return {nullptr, nullptr};
    return {reinterpret_cast<GetCurrentFn>(a), reinterpret_cast<GetIdFn>(b)};
  }();
  if (!fns.first || !fns.second) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (fns.first(&ctx) != CUDA_SUCCESS || !ctx || fns.second(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_noalloc_scratch in the current device's context.  It
// is looked up (cudaGetSymbolAddress, with the device current; no
// allocation) on the first call in a context and cached together with that
// context's id, so a later call from another context, or after the device
// was reset, looks it up again instead of reusing an address of a context
// that no longer exists.  Without context ids it is looked up on every call.
void* noalloc_scratch() {
  struct Entry {
    unsigned long long ctx;
    void* addr;
  };
  static std::mutex mu;
  static Entry cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (cudaSetDevice(dev) != cudaSuccess) return nullptr;  // makes the device's primary context current
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(mu);
  if (ctx != 0 && cache[dev].ctx == ctx && cache[dev].addr) return cache[dev].addr;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
  cache[dev] = Entry{ctx, p};
  return p;
}

// ---------------------------------------------------------------- decode
struct DecWs {
  size_t lse, total;
};
// Balanced mode runs at most this many CTAs (one per SM, B200 has 148).
constexpr int kDecGridMax = 1024;

// Partial results: rows * n_splits of them, or in balanced mode (n_splits =
// 0) one per (cache, CTA) slot and query head of its group: at most
// (B * Hkv + grid) * group <= B * Hq + kDecGridMax * 16 (group <= 16).
DecWs dec_layout(long long rows, int n_splits, int D) {  // rows = B * Hq
  const long long parts = n_splits > 0 ? rows * n_splits : rows + (long long)kDecGridMax * 16;
  const size_t o_bytes = up256((size_t)parts * D * 4);
  return {o_bytes, o_bytes + up256((size_t)parts * 4)};
}

// Split count for B * Hkv cache streams of up to L_max keys: the fewest
// splits that give about 0.8 x sm_count CTAs (one CTA fills an SM's shared
// memory), at most 64 and at least 256 keys each.  Longer key ranges per CTA
// amortise its start-up and the partial-result write; more than one wave only
// adds those costs (measured on B200 over 1..64 splits for group sizes 1, 4
// and 16, 1 to 64 sequences and 1K to 32K keys).
int dec_splits(long long units, int L_max) {
  if (units <= 0 || L_max <= 0) return 1;
  const long long tiles = (L_max + 31) / 32, target = (8 * sm_count() + 9) / 10;
  const long long nmax = std::max(1LL, std::min(64LL, tiles / 8));
  return (int)std::max(1LL, std::min(nmax, (target + units - 1) / units));
}

// Clusters of 2 to 4 CTAs merge in-kernel when all CTAs fit in one wave.
// Larger clusters, or several waves of them, measured slower on B200 than
// the separate merge launch: a cluster of 197 KB CTAs needs that many free
// SMs of one GPC at once, and its CTAs wait for its slowest one.
constexpr int kDecClusterMax = 4;

template <int D, bool BF16>
fa_status launch_decode_t(const fa::DecParams& p, cudaStream_t st) {
  using C = fa::DecCfg<D>;
  // caches as [B * Hkv, L, D]; 32-row boxes (L < 32 means no whole tile, so
  // the box is never used and only has to be valid)
  CUtensorMap mk, mv;
  const long long heads = (long long)p.B * p.Hkv;
  const int rows = std::max(p.L, 1);
  const unsigned box = (unsigned)std::min(C::KT, rows);
  if (!make_map(&mk, p.k, D, rows, heads, BF16, box) || !make_map(&mv, p.v, D, rows, heads, BF16, box))
    return FA_ERR_CUDA;
  if (set_smem<fa::decode_split_kernel<D, BF16>>(C::SMEM) != cudaSuccess) return FA_ERR_CUDA;
  cudaError_t e;
  if (p.n_splits == 0) {
    // balanced mode: the caches' tiles over one CTA per SM, then the merge
    if (set_smem<fa::decode_balanced_kernel<D, BF16>>(C::SMEM) != cudaSuccess) return FA_ERR_CUDA;
    fa::decode_balanced_kernel<D, BF16><<<(unsigned)p.grid, 128, C::SMEM, st>>>(mk, mv, p);
    g_launches.fetch_add(1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return from_cuda(e);
  } else {
    const long long ctas = (long long)p.n_splits * p.Hkv * p.B;
    if (p.n_splits >= 2 && p.n_splits <= kDecClusterMax && ctas <= sm_count()) {
      // the splits of one (sequence, KV head) as one cluster, merged in-kernel
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(p.n_splits, p.Hkv, p.B);
      cfg.blockDim = dim3(128);
      cfg.dynamicSmemBytes = C::SMEM;
      cfg.stream = st;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = p.n_splits;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      e = cudaLaunchKernelEx(&cfg, fa::decode_split_kernel<D, BF16>, mk, mv, p);
      g_launches.fetch_add(1);
      return from_cuda(e);
    }
    fa::decode_split_kernel<D, BF16><<<dim3(p.n_splits, p.Hkv, p.B), 128, C::SMEM, st>>>(mk, mv, p);
    g_launches.fetch_add(1);
    e = cudaGetLastError();
    if (e != cudaSuccess || p.n_splits == 1) return from_cuda(e);  // one split writes O and LSE itself
  }
  // the merge as a programmatic dependent launch: it is scheduled while the
  // split kernel runs and waits (griddepcontrol.wait) for its results
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((long long)p.B * p.Hq));
  cfg.blockDim = dim3(D);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, fa::decode_merge_kernel<D, BF16>, p);
  g_launches.fetch_add(1);
  return from_cuda(e);
}

// ---------------------------------------------------------------- dropout
// 16-bit keep threshold t = max(1, floor((1 - p) 2^16)) and scale 2^16 / t
// (the inverse of the exact keep probability t / 2^16); p in (0, 1).
fa::Dropout make_dropout(float p, uint64_t seed, uint64_t offset) {
  fa::Dropout d;
  const double t = std::max(1.0, std::floor((1.0 - (double)p) * 256.0));
  d.thresh = (uint32_t)t;
  d.seed_lo = (uint32_t)seed;
  d.seed_hi = (uint32_t)(seed >> 32);
  d.offset = (uint32_t)offset;
  d.scale = (float)(256.0 / t);
  return d;
}

bool dropout_p_ok(float p) { return std::isfinite(p) && p >= 0.f && p < 1.f; }

}  // namespace

extern "C" {

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int S, int D,
                 float scale, int causal, fa_dtype dt, void* stream) {
  if (B < 0 || H < 0 || S < 0) return FA_ERR_INVALID_ARG;
  if (dt != FA_BF16 && dt != FA_FP16) return FA_ERR_INVALID_ARG;
  if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || S == 0) return FA_OK;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_INVALID_ARG;
  const long long heads = (long long)B * H;
  if (heads > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  return run_fwd(q, k, v, o, lse, nullptr, (int)heads, S, S, 1, D, scale, causal != 0, dt == FA_BF16, false,
                 static_cast<cudaStream_t>(stream));
}

fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens,
                        int nseq, int max_seqlen, int total, int H, int D, float scale, int causal, fa_dtype dt,
                        void* stream) {
  if (nseq < 0 || max_seqlen < 0 || total < 0 || H < 0) return FA_ERR_INVALID_ARG;
  if (dt != FA_BF16 && dt != FA_FP16) return FA_ERR_INVALID_ARG;
  if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (nseq == 0 || H == 0 || total == 0 || max_seqlen == 0) return FA_OK;
  if (max_seqlen > total) return FA_ERR_INVALID_ARG;
  if (!q || !k || !v || !o || !lse || !cu_seqlens) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return FA_ERR_INVALID_ARG;
  return run_fwd(q, k, v, o, lse, cu_seqlens, H, max_seqlen, total, nseq, D, scale, causal != 0, dt == FA_BF16, true,
                 static_cast<cudaStream_t>(stream));
}

size_t fa_bwd_workspace_size(int B, int H, int S, int D) {
  if (B <= 0 || H <= 0 || S <= 0 || (D != 64 && D != 128)) return 0;
  return ws_layout((long long)B * H, 1, S, S, D).total;
}

fa_status fa_bwd_preprocess(const void* o, const void* dO, const float* lse, int B, int H, int S, int D,
                            fa_dtype dt, void* workspace, size_t workspace_bytes, void* stream) {
  fa_status c = bwd_common_checks(B, H, S, D, dt, workspace, workspace_bytes);
  if (c != FA_OK || B == 0 || H == 0 || S == 0) return c;
  if (!ptrs_ok({o, dO, lse})) return FA_ERR_INVALID_ARG;
  const fa::BwdParams p =
      bwd_params(B * H, 1, S, S, nullptr, D, 1.f, 0, static_cast<uint8_t*>(workspace), nullptr, nullptr);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (D == 64)
    return dt == FA_BF16 ? launch_bwd_pre<64, true>(o, dO, lse, p, false, st)
                         : launch_bwd_pre<64, false>(o, dO, lse, p, false, st);
  return dt == FA_BF16 ? launch_bwd_pre<128, true>(o, dO, lse, p, false, st)
                       : launch_bwd_pre<128, false>(o, dO, lse, p, false, st);
}

fa_status fa_bwd_main(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv, int B, int H,
                      int S, int D, float scale, int causal, fa_dtype dt, int deterministic, void* workspace,
                      size_t workspace_bytes, void* stream) {
  fa_status c = bwd_common_checks(B, H, S, D, dt, workspace, workspace_bytes);
  if (c != FA_OK) return c;
  if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || S == 0) return FA_OK;
  if (!ptrs_ok({q, k, v, dO, dk, dv})) return FA_ERR_INVALID_ARG;
  const fa::BwdParams p = bwd_params(B * H, 1, S, S, nullptr, D, scale, deterministic != 0,
                                     static_cast<uint8_t*>(workspace), dk, dv);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool cz = causal != 0;
  if (D == 64)
    return dt == FA_BF16 ? launch_bwd_main<64, true>(q, k, v, dO, p, cz, false, false, st)
                         : launch_bwd_main<64, false>(q, k, v, dO, p, cz, false, false, st);
  return dt == FA_BF16 ? launch_bwd_main<128, true>(q, k, v, dO, p, cz, false, false, st)
                       : launch_bwd_main<128, false>(q, k, v, dO, p, cz, false, false, st);
}

fa_status fa_bwd_finish(void* dq, int B, int H, int S, int D, float scale, fa_dtype dt, int deterministic,
                        void* workspace, size_t workspace_bytes, void* stream) {
  fa_status c = bwd_common_checks(B, H, S, D, dt, workspace, workspace_bytes);
  if (c != FA_OK) return c;
  if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || S == 0) return FA_OK;
  if (!ptrs_ok({dq})) return FA_ERR_INVALID_ARG;
  const fa::BwdParams p =
      bwd_params(B * H, 1, S, S, nullptr, D, scale, 0, static_cast<uint8_t*>(workspace), nullptr, nullptr);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dt == FA_BF16 ? launch_bwd_post<true>(dq, p, D, st, deterministic != 0)
                       : launch_bwd_post<false>(dq, p, D, st, deterministic != 0);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                 void* dq, void* dk, void* dv, int B, int H, int S, int D, float scale, int causal, fa_dtype dt,
                 int deterministic, void* workspace, size_t workspace_bytes, void* stream) {
  fa_status c = bwd_common_checks(B, H, S, D, dt, workspace, workspace_bytes);
  if (c != FA_OK) return c;
  if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || S == 0) return FA_OK;
  if (!ptrs_ok({q, k, v, o, dO, lse, dq, dk, dv})) return FA_ERR_INVALID_ARG;
  c = fa_bwd_preprocess(o, dO, lse, B, H, S, D, dt, workspace, workspace_bytes, stream);
  if (c != FA_OK) return c;
  c = fa_bwd_main(q, k, v, dO, dk, dv, B, H, S, D, scale, causal, dt, deterministic, workspace, workspace_bytes,
                  stream);
  if (c != FA_OK) return c;
  return fa_bwd_finish(dq, B, H, S, D, scale, dt, deterministic, workspace, workspace_bytes, stream);
}

fa_status fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int S,
                         int D, float scale, int causal, fa_dtype dt, float dropout_p, uint64_t seed,
                         uint64_t offset, void* stream) {
  if (!dropout_p_ok(dropout_p)) return FA_ERR_INVALID_ARG;
  if (dropout_p == 0.f) return fa_fwd(q, k, v, o, lse, B, H, S, D, scale, causal, dt, stream);
  if (B < 0 || H < 0 || S < 0) return FA_ERR_INVALID_ARG;
  if (dt != FA_BF16 && dt != FA_FP16) return FA_ERR_INVALID_ARG;
  if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || S == 0) return FA_OK;
  if (!ptrs_ok({q, k, v, o, lse})) return FA_ERR_INVALID_ARG;
  const long long heads = (long long)B * H;
  if (heads > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  const fa::Dropout d = make_dropout(dropout_p, seed, offset);
  return run_fwd(q, k, v, o, lse, nullptr, (int)heads, S, S, 1, D, scale, causal != 0, dt == FA_BF16, false,
                 static_cast<cudaStream_t>(stream), &d);
}

fa_status fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                         void* dq, void* dk, void* dv, int B, int H, int S, int D, float scale, int causal,
                         fa_dtype dt, int deterministic, float dropout_p, uint64_t seed, uint64_t offset,
                         void* workspace, size_t workspace_bytes, void* stream) {
  if (!dropout_p_ok(dropout_p)) return FA_ERR_INVALID_ARG;
  if (dropout_p == 0.f)
    return fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, S, D, scale, causal, dt, deterministic, workspace,
                  workspace_bytes, stream);
  fa_status c = bwd_common_checks(B, H, S, D, dt, workspace, workspace_bytes);
  if (c != FA_OK) return c;
  if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || S == 0) return FA_OK;
  if (!ptrs_ok({q, k, v, o, dO, lse, dq, dk, dv})) return FA_ERR_INVALID_ARG;
  fa::BwdParams p = bwd_params(B * H, 1, S, S, nullptr, D, scale, deterministic != 0,
                               static_cast<uint8_t*>(workspace), dk, dv);
  p.drop = make_dropout(dropout_p, seed, offset);
  return run_bwd(q, k, v, o, dO, lse, dq, p, D, causal != 0, dt == FA_BF16, false, static_cast<cudaStream_t>(stream),
                 true);
}

fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                         const float* lse, void* dq, void* dk, void* dv, int B, int H, int S, int D, float scale,
                         int causal, fa_dtype dt, int deterministic, void* stream) {
  if (B < 0 || H < 0 || S < 0) return FA_ERR_INVALID_ARG;
  if (dt != FA_BF16 && dt != FA_FP16) return FA_ERR_INVALID_ARG;
  if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || S == 0) return FA_OK;
  if ((long long)B * H > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  if (!ptrs_ok({q, k, v, o, dO, lse, dq, dk, dv})) return FA_ERR_INVALID_ARG;
  // sizes whose scratch does not fit the fixed array are refused up front
  if (fa_bwd_workspace_size(B, H, S, D) > (size_t)FA_BWD_NOALLOC_SCRATCH_BYTES) return FA_ERR_UNSUPPORTED;
  void* scratch = noalloc_scratch();
  if (!scratch) return FA_ERR_CUDA;
  return fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, S, D, scale, causal, dt, deterministic, scratch,
                (size_t)FA_BWD_NOALLOC_SCRATCH_BYTES, stream);
}

fa_status fa_fwd_varlen_dropout(const void* q, const void* k, const void* v, void* o, float* lse,
                                const int* cu_seqlens, int nseq, int max_seqlen, int total, int H, int D, float scale,
                                int causal, fa_dtype dt, float dropout_p, uint64_t seed, uint64_t offset,
                                void* stream) {
  if (!dropout_p_ok(dropout_p)) return FA_ERR_INVALID_ARG;
  if (dropout_p == 0.f)
    return fa_fwd_varlen(q, k, v, o, lse, cu_seqlens, nseq, max_seqlen, total, H, D, scale, causal, dt, stream);
  if (nseq < 0 || max_seqlen < 0 || total < 0 || H < 0) return FA_ERR_INVALID_ARG;
  if (dt != FA_BF16 && dt != FA_FP16) return FA_ERR_INVALID_ARG;
  if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (nseq == 0 || H == 0 || total == 0 || max_seqlen == 0) return FA_OK;
  if (max_seqlen > total) return FA_ERR_INVALID_ARG;
  if (!ptrs_ok({q, k, v, o, lse}) || !cu_seqlens || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return FA_ERR_INVALID_ARG;
  if ((long long)nseq * H > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  const fa::Dropout d = make_dropout(dropout_p, seed, offset);
  return run_fwd(q, k, v, o, lse, cu_seqlens, H, max_seqlen, total, nseq, D, scale, causal != 0, dt == FA_BF16, true,
                 static_cast<cudaStream_t>(stream), &d);
}

size_t fa_bwd_varlen_workspace_size(int nseq, int max_seqlen, int total, int H, int D) {
  if (nseq <= 0 || max_seqlen <= 0 || total <= 0 || H <= 0 || (D != 64 && D != 128)) return 0;
  return ws_layout(H, nseq, max_seqlen, total, D).total;
}

fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dO,
                        const float* lse, void* dq, void* dk, void* dv, const int* cu_seqlens, int nseq,
                        int max_seqlen, int total, int H, int D, float scale, int causal, fa_dtype dt,
                        int deterministic, void* workspace, size_t workspace_bytes, void* stream) {
  if (nseq < 0 || max_seqlen < 0 || total < 0 || H < 0) return FA_ERR_INVALID_ARG;
  if (dt != FA_BF16 && dt != FA_FP16) return FA_ERR_INVALID_ARG;
  if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (nseq == 0 || H == 0 || total == 0 || max_seqlen == 0) return FA_OK;
  if (max_seqlen > total) return FA_ERR_INVALID_ARG;
  if (!ptrs_ok({q, k, v, o, dO, lse, dq, dk, dv}) || !cu_seqlens || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return FA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return FA_ERR_INVALID_ARG;
  if (workspace_bytes < ws_layout(H, nseq, max_seqlen, total, D).total) return FA_ERR_INVALID_ARG;
  const fa::BwdParams p = bwd_params(H, nseq, max_seqlen, total, cu_seqlens, D, scale, deterministic != 0,
                                     static_cast<uint8_t*>(workspace), dk, dv);
  return run_bwd(q, k, v, o, dO, lse, dq, p, D, causal != 0, dt == FA_BF16, true, static_cast<cudaStream_t>(stream));
}

fa_status fa_bwd_varlen_dropout(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                const float* lse, void* dq, void* dk, void* dv, const int* cu_seqlens, int nseq,
                                int max_seqlen, int total, int H, int D, float scale, int causal, fa_dtype dt,
                                int deterministic, float dropout_p, uint64_t seed, uint64_t offset, void* workspace,
                                size_t workspace_bytes, void* stream) {
  if (!dropout_p_ok(dropout_p)) return FA_ERR_INVALID_ARG;
  if (dropout_p == 0.f)
    return fa_bwd_varlen(q, k, v, o, dO, lse, dq, dk, dv, cu_seqlens, nseq, max_seqlen, total, H, D, scale, causal,
                         dt, deterministic, workspace, workspace_bytes, stream);
  if (nseq < 0 || max_seqlen < 0 || total < 0 || H < 0) return FA_ERR_INVALID_ARG;
  if (dt != FA_BF16 && dt != FA_FP16) return FA_ERR_INVALID_ARG;
  if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (nseq == 0 || H == 0 || total == 0 || max_seqlen == 0) return FA_OK;
  if (max_seqlen > total) return FA_ERR_INVALID_ARG;
  if (!ptrs_ok({q, k, v, o, dO, lse, dq, dk, dv}) || !cu_seqlens || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return FA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return FA_ERR_INVALID_ARG;
  if (workspace_bytes < ws_layout(H, nseq, max_seqlen, total, D).total) return FA_ERR_INVALID_ARG;
  fa::BwdParams p = bwd_params(H, nseq, max_seqlen, total, cu_seqlens, D, scale, deterministic != 0,
                               static_cast<uint8_t*>(workspace), dk, dv);
  p.drop = make_dropout(dropout_p, seed, offset);
  return run_bwd(q, k, v, o, dO, lse, dq, p, D, causal != 0, dt == FA_BF16, true, static_cast<cudaStream_t>(stream),
                 true);
}

int fa_decode_num_splits(int B, int Hkv, int L_max) {
  if (B <= 0 || Hkv <= 0 || L_max <= 0) return 1;
  return dec_splits((long long)B * Hkv, L_max);
}

size_t fa_decode_workspace_size(int B, int Hq, int n_splits, int D) {
  if (B <= 0 || Hq <= 0 || n_splits < 0 || n_splits > 1024 || (D != 64 && D != 128)) return 0;
  return dec_layout((long long)B * Hq, n_splits, D).total;
}

fa_status fa_decode(const void* q, const void* k_cache, const void* v_cache, const int* seq_lens, void* o, float* lse,
                    int B, int Hq, int Hkv, int L_max, int D, float scale, fa_dtype dt, int n_splits, void* workspace,
                    size_t workspace_bytes, void* stream) {
  if (B < 0 || Hq < 0 || Hkv < 0 || L_max < 0) return FA_ERR_INVALID_ARG;
  if (dt != FA_BF16 && dt != FA_FP16) return FA_ERR_INVALID_ARG;
  if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (B == 0 || Hq == 0) return FA_OK;
  if (Hkv == 0 || Hq % Hkv) return FA_ERR_INVALID_ARG;
  if (Hq / Hkv > 16) return FA_ERR_UNSUPPORTED;
  if (n_splits < 0 || n_splits > 1024) return FA_ERR_INVALID_ARG;
  if (B > 65535 || Hkv > 65535 || (long long)B * Hq > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  if (!ptrs_ok({q, k_cache, v_cache, o, lse}) || !seq_lens || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return FA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return FA_ERR_INVALID_ARG;
  const DecWs w = dec_layout((long long)B * Hq, n_splits, D);
  if (workspace_bytes < w.total) return FA_ERR_INVALID_ARG;
  fa::DecParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.k = static_cast<const uint16_t*>(k_cache);
  p.v = static_cast<const uint16_t*>(v_cache);
  p.seq_lens = seq_lens;
  p.o_part = reinterpret_cast<float*>(workspace);
  p.lse_part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + w.lse);
  p.o = o;
  p.lse = lse;
  p.B = B, p.Hq = Hq, p.Hkv = Hkv, p.L = L_max, p.n_splits = n_splits, p.group = Hq / Hkv;
  p.tpp = std::max(1, (L_max + fa::DecCfg<64>::KT - 1) / fa::DecCfg<64>::KT);
  p.tiles = (long long)B * Hkv * p.tpp;
  p.grid = (int)std::min<long long>(std::min(sm_count(), kDecGridMax), p.tiles);
  p.scale_log2 = scale * 1.4426950408889634f;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (D == 128) return dt == FA_BF16 ? launch_decode_t<128, true>(p, st) : launch_decode_t<128, false>(p, st);
  return dt == FA_BF16 ? launch_decode_t<64, true>(p, st) : launch_decode_t<64, false>(p, st);
}

fa_status fa_selftest_timeout(void* stream) {
  selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  g_launches.fetch_add(1);
  return from_cuda(cudaGetLastError());
}

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: null, misaligned or out-of-range argument";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: head dim or size not implemented";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: a CUDA call failed";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a kernel gave up waiting on an internal barrier";
  }
  return "unknown fa_status";
}

fa_status fa_check_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  uint32_t code = 0;
  if (cudaMemcpyFromSymbol(&code, fa::g_dev_error, sizeof(code)) != cudaSuccess) return FA_ERR_CUDA;
  if (code == 0) return FA_OK;
  const uint32_t zero = 0;
  if (cudaMemcpyToSymbol(fa::g_dev_error, &zero, sizeof(zero)) != cudaSuccess) return FA_ERR_CUDA;
  return code == fa::DEV_ERR_ARG ? FA_ERR_INVALID_ARG : FA_ERR_TIMEOUT;
}

uint64_t fa_launch_count(void) { return g_launches.load(); }

}  // extern "C"

/*
 * fa.h - C ABI of the exact tiled attention library (libfa.so) for NVIDIA B200 (sm_100a).
 *
 * The library computes exact scaled dot-product attention
 *
 *     O = softmax(Q K^T * scale [+ causal mask]) V
 *
 * tile by tile with an online softmax, so the S x S score and probability
 * matrices never reach device memory ("From Self-Attention to FlashAttention",
 * §一 flowchart and §二 Online Softmax; "ops-transformer里的FlashAttention",
 * "FlashAttention的核心思路").  The forward keeps only the per-row log-sum-exp,
 * and the backward rebuilds each local probability block from it
 * ("Flash Attention 的算法设计原理", "核心机制", third item).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are dense, row-major, 16-bit (bf16 or fp16 as chosen by `dt`) in
 *    device memory owned by the caller.  The library never allocates,
 *    frees or keeps a pointer across calls.
 *  - Dense layout: [B, H, S, D] contiguous (D innermost).  LSE: fp32 [B, H, S].
 *  - Packed variable-length layout: [H, T, D] contiguous, T = total tokens;
 *    sequence s occupies token rows cu_seqlens[s] .. cu_seqlens[s+1]-1.
 *    LSE: fp32 [H, T].
 *  - Every base pointer must be 16-byte aligned (the kernels move tiles with
 *    the Tensor Memory Accelerator).
 *  - Supported head dims: D = 64 or 128.  S (or each sequence) may be any
 *    length >= 1; ragged tails are handled inside the kernels.
 *  - causal != 0 lets query i attend keys j <= i (diagonal included, counted
 *    from the start of each sequence), as the causal flag of the operator in
 *    "ops-transformer里的FlashAttention", "ops-transformer里的完整算子" and
 *    "实战踩坑 坑二".
 *  - scale is applied to Q K^T (normally 1/sqrt(D)); it must be finite and > 0.
 *  - All calls are asynchronous on `stream` (a cudaStream_t, 0 = legacy
 *    default stream).  Argument errors are reported synchronously before
 *    anything is launched; launch failures return FA_ERR_CUDA.  A kernel that
 *    waits too long on one of its internal barriers gives up, records
 *    FA_ERR_TIMEOUT in a per-device error word and exits; read it with
 *    fa_check_device_error().
 *  - The compute calls may be recorded into a CUDA graph (stream capture)
 *    once one call of the same kind has run outside the capture on the device
 *    (it sets up per-device state); a replay reads the buffers as they are
 *    then.  fa_check_device_error() synchronises and must stay outside.
 *  - No entry point falls back to another implementation: unsupported
 *    arguments return FA_ERR_UNSUPPORTED.
 */
#ifndef EXACT_TILED_ATTENTION_FA_H
#define EXACT_TILED_ATTENTION_FA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, negative size, bad scale */
  FA_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. D not in {64,128}) */
  FA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
  FA_ERR_TIMEOUT = 4      /* a kernel gave up waiting on an internal barrier */
} fa_status;

typedef enum { FA_BF16 = 0, FA_FP16 = 1 } fa_dtype;

/*
 * Forward pass.
 *   q, k, v : [B, H, S, D] inputs (read only).
 *   o       : [B, H, S, D] output, same dtype.
 *   lse     : [B, H, S] fp32 output, natural-log log-sum-exp of each row's
 *             scaled scores (the statistic the backward recomputes P from).
 * Cites: "From Self-Attention to FlashAttention", §二 (running max / running
 * sum update, final division); "ops-transformer里的FlashAttention",
 * "核心计算流程" (Q tile resident, K/V tiles streamed, only O written back).
 * B, H or S equal to 0 is a no-op returning FA_OK.
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int H, int S, int D, float scale, int causal, fa_dtype dt,
                 void* stream);

/*
 * Forward pass over a packed batch of variable-length sequences.
 *   q, k, v, o : [H, total, D];  lse : fp32 [H, total].
 *   cu_seqlens : DEVICE int32 [nseq + 1], cu_seqlens[0] = 0, non-decreasing,
 *                cu_seqlens[nseq] = total.
 *   max_seqlen : an upper bound on every sequence length (sizes the grid).
 * Each sequence attends only within itself.  Cites: "Flash Attention 的算法设计原理",
 * "练习口述回答" (variable-length inputs are a branch to cover on their own).
 * The library does not read cu_seqlens on the host; offsets that break the
 * stated rules give unspecified (but in-bounds) results.
 */
fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                        const int* cu_seqlens, int nseq, int max_seqlen, int total,
                        int H, int D, float scale, int causal, fa_dtype dt, void* stream);

/*
 * Bytes of device scratch that fa_bwd needs for these sizes: two fp32 dQ
 * accumulators [B, H, S, D] (the second holds the odd key tiles' sums in
 * deterministic mode), one 32-byte row per query (LSE and the row term
 * D_i = dO_i . O_i, as bf16 parts, rows padded to multiples of 128), the
 * ordering counters of deterministic mode (two per query tile) and the work
 * counter of the backward's persistent grid, each 256-byte aligned.
 * Returns 0 for unsupported sizes.
 * This is the first half of the two-phase call of the operator in
 * "ops-transformer里的FlashAttention", "ops-transformer里的完整算子": a size
 * query for the workspace (there aclnnFlashAttentionGetWorkspaceSize), then
 * the computation given a caller-allocated workspace of that size.
 */
size_t fa_bwd_workspace_size(int B, int H, int S, int D);

/*
 * Backward pass.  Inputs q, k, v, o, dO ([B, H, S, D]) and lse ([B, H, S],
 * from fa_fwd); outputs dq, dk, dv ([B, H, S, D], same dtype).
 * workspace: caller-owned device buffer of at least
 * fa_bwd_workspace_size(B, H, S, D) bytes, 256-byte aligned; its contents on
 * entry do not matter and are overwritten.
 * deterministic = 0: dQ partial sums from different key tiles are added with
 *   fp32 reductions (TMA bulk reduce-adds) in whatever order the key tiles
 *   reach them, so dq may differ in the last bits from run to run.
 * deterministic = 1: the dQ partials of one query tile are added in a fixed
 *   order: the even key tiles into one fp32 accumulator and the odd ones
 *   into another, each from the highest key tile down, and the two sums are
 *   added at the end, so repeated calls with the same inputs, sizes and GPU
 *   give bit-identical dq (the `deterministic` option of the operator config
 *   in "ops-transformer里的FlashAttention", "ops-transformer里的完整算子").
 * The gradients are those of L = sum(dO * O): dV = P^T dO, dS = P o (dP - D),
 * dQ = scale dS K, dK = scale dS^T Q, with P rebuilt from lse
 * ("Flash Attention 的算法设计原理", "核心机制"; the pages print no formulas, these
 * are the textbook ones).
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                 const float* lse, void* dq, void* dk, void* dv,
                 int B, int H, int S, int D, float scale, int causal, fa_dtype dt,
                 int deterministic, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward pass over a packed batch of variable-length sequences (the
 * gradients of fa_fwd_varlen's output; same formulas as fa_bwd, each
 * sequence on its own, causal counted from its first token).
 *   q, k, v, o, dO : [H, total, D];  lse : fp32 [H, total] from fa_fwd_varlen.
 *   dq, dk, dv     : [H, total, D] outputs, same dtype.
 *   cu_seqlens, nseq, max_seqlen, total : as for fa_fwd_varlen.
 *   workspace : caller-owned device buffer of at least
 *               fa_bwd_varlen_workspace_size(nseq, max_seqlen, total, H, D)
 *               bytes, 256-byte aligned; contents on entry do not matter.
 *   deterministic : as for fa_bwd (key tiles of one sequence add into a query
 *               tile in increasing order).
 * Cites: "Flash Attention 的算法设计原理", "练习口述回答" (variable-length inputs
 * are a branch to test on their own) and "核心机制" (recompute P from the
 * saved statistics).  nseq, H, total or max_seqlen equal to 0 is a no-op.
 */
/* Workspace size query of fa_bwd_varlen: the same two-phase call as
 * fa_bwd_workspace_size ("ops-transformer里的完整算子"); 0 for unsupported sizes. */
size_t fa_bwd_varlen_workspace_size(int nseq, int max_seqlen, int total, int H, int D);
fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dO,
                        const float* lse, void* dq, void* dk, void* dv,
                        const int* cu_seqlens, int nseq, int max_seqlen, int total,
                        int H, int D, float scale, int causal, fa_dtype dt,
                        int deterministic, void* workspace, size_t workspace_bytes, void* stream);

/*
 * The three launches fa_bwd makes (the pages describe the backward as one
 * operator; the split only exposes its phases), exposed for callers that want to place
 * or time them separately (same arguments, same rules, same workspace; they
 * must run in this order on one stream):
 *   fa_bwd_preprocess  D_i = dO_i . O_i and LSE into the workspace (as
 *                      the per-query rows of an extra product step);
 *                      clears the dQ accumulator, the deterministic-mode
 *                      counters and the work counter fa_bwd_main claims
 *                      its units from.
 *   fa_bwd_main        the tiled pass over key/value tiles: writes dk, dv
 *                      and accumulates unscaled dQ (fp32) in the workspace.
 *   fa_bwd_finish      dq = scale * accumulated dQ (the sum of both
 *                      accumulators when deterministic), rounded to the
 *                      dtype.  `deterministic` must be the value given to
 *                      fa_bwd_main; the kernel compares it with the mark
 *                      fa_bwd_main left in the workspace and, when they
 *                      differ, records an argument error that
 *                      fa_check_device_error() returns as FA_ERR_INVALID_ARG
 *                      (dq is then wrong).
 */
fa_status fa_bwd_preprocess(const void* o, const void* dO, const float* lse, int B, int H, int S, int D,
                            fa_dtype dt, void* workspace, size_t workspace_bytes, void* stream);
fa_status fa_bwd_main(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv,
                      int B, int H, int S, int D, float scale, int causal, fa_dtype dt, int deterministic,
                      void* workspace, size_t workspace_bytes, void* stream);
fa_status fa_bwd_finish(void* dq, int B, int H, int S, int D, float scale, fa_dtype dt, int deterministic,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward pass that allocates nothing and takes no workspace.
 *
 * Some callers cannot call cudaMalloc: code that runs inside a device memory
 * allocator's own hooks (a nested allocation would re-enter it), processes
 * whose device memory is planned up front and must not grow while they run,
 * and latency-critical loops where an allocation may stall on the device.
 * For them, fa_bwd_noalloc computes exactly what fa_bwd computes (same
 * arguments, same results, same deterministic option) but keeps its scratch
 * (the fp32 dQ accumulator, the D_i and LSE rows, the ordering counters) in
 * one fixed array of FA_BWD_NOALLOC_SCRATCH_BYTES bytes that lives in device
 * memory from the moment the library is loaded on a device until the
 * process exits.  The caller still provides every input and output.
 *   - Sizes with fa_bwd_workspace_size(B, H, S, D) > FA_BWD_NOALLOC_SCRATCH_BYTES
 *     are refused with FA_ERR_UNSUPPORTED before anything is launched.
 *   - The first call in each device context looks up that array's device
 *     address (with the device current) and caches it with the context's
 *     process-unique id; make that first call before any stream capture.
 *     A call from another context, or after cudaDeviceReset, looks the
 *     address up again rather than reuse one of a context that is gone.
 *   - Every call on a device shares the one array, which keeps the previous
 *     call's contents; each call clears what must start at zero itself.
 *     Calls whose kernels overlap on the GPU (different streams without
 *     ordering between them) race on the array: serialise them.
 *   - It never calls cudaMalloc, cudaFree or any allocating library routine.
 * The pages describe no such variant; it exists for the callers above.
 */
#define FA_BWD_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                         const float* lse, void* dq, void* dk, void* dv,
                         int B, int H, int S, int D, float scale, int causal, fa_dtype dt,
                         int deterministic, void* stream);

/*
 * Dropout on the attention probabilities (dense [B, H, S, D] batches; packed
 * batches below).
 * "Flash Attention 的算法设计原理", section "练习口述回答", lists dropout as a
 * branch to test on its own. Because the mask must be regenerated in the
 * backward rather than stored, it comes from a counter-based generator.
 *
 *   O   = (P * M * s) V,  P = softmax(Q K^T scale [+ causal]),
 *   LSE = that of the undropped P (as fa_fwd).
 *
 * The mask M[b,h,i,j] comes from Philox4x32-10 (Salmon et al., "Parallel
 * random numbers: as easy as 1, 2, 3", SC 2011):
 *   - counter (j >> 3, i >> 1, b*H + h, offset mod 2^32);
 *   - key (seed mod 2^32, seed >> 32);
 *   - word 2*(i & 1) + ((j >> 2) & 1), byte j & 3 of it (bits 8(j & 3) ..).
 * M = 1 when that byte is below t = max(1, floor((1 - p) * 2^8)).
 * An element is therefore kept with probability t / 2^8 (dropout_p is taken
 * to the smallest multiple of 2^-8 that is not below it), and s = 2^8 / t
 * keeps E[O] exact.
 * fa_bwd_dropout, given the same (dropout_p, seed, offset), regenerates M.
 * It returns the gradients of sum(dO * O) for that O:
 *   dV = (P*M*s)^T dO
 *   dS = P * (dO V^T * M*s - D),  D_i = dO_i . O_i
 *   dQ = scale dS K,  dK = scale dS^T Q
 *
 * Every argument is that of fa_fwd / fa_bwd, plus dropout_p in [0, 1),
 * seed and offset. Anything else returns FA_ERR_INVALID_ARG. dropout_p = 0
 * is exactly fa_fwd / fa_bwd. The workspace is that of
 * fa_bwd_workspace_size(B, H, S, D).
 */
fa_status fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int S,
                         int D, float scale, int causal, fa_dtype dt, float dropout_p, uint64_t seed,
                         uint64_t offset, void* stream);
fa_status fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o, const void* dO,
                         const float* lse, void* dq, void* dk, void* dv, int B, int H, int S, int D, float scale,
                         int causal, fa_dtype dt, int deterministic, float dropout_p, uint64_t seed,
                         uint64_t offset, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Dropout on a packed batch of variable-length sequences: fa_fwd_varlen /
 * fa_bwd_varlen with the dropout of fa_fwd_dropout / fa_bwd_dropout.  The
 * pages name both branches ("Flash Attention 的算法设计原理", "练习口述回答") but
 * no mask layout for a pack; sequence s takes the mask that batch index s of
 * a dense batch would get (the counter's head word is s * H + h, query and
 * key indices count from the sequence's first token), so a pack of equal
 * lengths drops exactly what the dense [nseq, H, L, D] batch drops.
 * Arguments: those of fa_fwd_varlen / fa_bwd_varlen plus dropout_p, seed,
 * offset as for fa_fwd_dropout; dropout_p = 0 is exactly the plain call.
 */
fa_status fa_fwd_varlen_dropout(const void* q, const void* k, const void* v, void* o, float* lse,
                                const int* cu_seqlens, int nseq, int max_seqlen, int total, int H, int D,
                                float scale, int causal, fa_dtype dt, float dropout_p, uint64_t seed,
                                uint64_t offset, void* stream);
fa_status fa_bwd_varlen_dropout(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                const float* lse, void* dq, void* dk, void* dv, const int* cu_seqlens, int nseq,
                                int max_seqlen, int total, int H, int D, float scale, int causal, fa_dtype dt,
                                int deterministic, float dropout_p, uint64_t seed, uint64_t offset, void* workspace,
                                size_t workspace_bytes, void* stream);

/*
 * Decode: one new query token per (sequence, query head) against a KV cache
 * ("Flash Attention 的算法设计原理", sections "训练与推理价值" and "练习口述回答":
 * at inference the new token reads the whole, growing cache, and GQA/MQA
 * share one KV head among several query heads).  For b < B, h < Hq:
 *
 *   O[b,h,:]  = softmax(q[b,h,:] . K[b,h/G,j,:] * scale, j < len_b) V[b,h/G,:,:]
 *   lse[b,h]  = log sum_{j < len_b} exp(q[b,h,:] . K[b,h/G,j,:] * scale)
 *
 * with G = Hq / Hkv and len_b = min(max(seq_lens[b], 0), L_max); every cached
 * key is visible (the new token is the last position).  len_b = 0 gives
 * O = 0 and lse = -inf.
 *
 *   q        [B, Hq, D] 16-bit (dt), contiguous
 *   k_cache, v_cache  [B, Hkv, L_max, D] 16-bit, contiguous; rows at or past
 *            len_b are never read
 *   seq_lens [B] int32 in device memory (4-byte aligned)
 *   o        [B, Hq, D] 16-bit (dt);  lse [B, Hq] fp32, natural log
 *   n_splits number of key ranges each cache is cut into (1..1024), or 0.
 *            Each range is reduced by its own CTA to a normalised partial O
 *            and its LSE, and the parts are merged:
 *            LSE = log sum_s exp(LSE_s), O = sum_s exp(LSE_s - LSE) O_s.
 *            One range writes O and LSE directly; 2 to 4 ranges whose CTAs
 *            fit in one wave merge inside the kernel (a thread-block cluster,
 *            through distributed shared memory); otherwise the parts go to
 *            the workspace and a second, dependent launch merges them.
 *            0 ("balanced"): one CTA per SM, each running an equal share of
 *            all caches' 32-key tiles (a share may end one cache and start
 *            the next), one part per cache it meets, merged by the second
 *            launch.  fa_decode_num_splits() returns the library's choice.
 *   workspace  device memory of at least fa_decode_workspace_size(B, Hq,
 *            n_splits, D) bytes, 256-byte aligned, owned by the caller; it
 *            may be reused once the call's work on `stream` has finished.
 *
 * Requirements: D = 64 or 128; Hkv >= 1 with Hq a multiple of Hkv
 * (FA_ERR_INVALID_ARG otherwise) and G = Hq / Hkv <= 16 (FA_ERR_UNSUPPORTED
 * otherwise); B, Hkv <= 65535; q, k_cache, v_cache, o, lse 16-byte aligned.
 * B = 0 or Hq = 0 is a no-op.  One or two kernel launches on `stream`.
 */
/* The library's split count for fa_decode at these sizes (the key ranges of
 * "训练与推理价值"'s decode over a long cache; the pages give no rule, this one
 * is measured on B200). */
int fa_decode_num_splits(int B, int Hkv, int L_max);
/* Workspace bytes for fa_decode with these sizes: fp32 partial O and LSE per
 * (sequence, query head, part); n_splits = 0 sizes balanced mode (B * Hq +
 * 16384 part slots, independent of the cache length).  0 for unsupported
 * arguments.  The two-phase size query of "ops-transformer里的FlashAttention",
 * "ops-transformer里的完整算子". */
size_t fa_decode_workspace_size(int B, int Hq, int n_splits, int D);
fa_status fa_decode(const void* q, const void* k_cache, const void* v_cache, const int* seq_lens, void* o,
                    float* lse, int B, int Hq, int Hkv, int L_max, int D, float scale, fa_dtype dt,
                    int n_splits, void* workspace, size_t workspace_bytes, void* stream);

/* A static, human-readable name for a status code.  No page defines status
 * codes; they are this library's error reporting. */
const char* fa_status_string(fa_status s);

/*
 * Synchronises `stream`, then reads and clears the calling device's error
 * word.  Returns FA_OK, FA_ERR_TIMEOUT (a kernel gave up waiting),
 * FA_ERR_INVALID_ARG (fa_bwd_finish was told another deterministic mode
 * than fa_bwd_main ran in) or FA_ERR_CUDA (the synchronisation itself
 * failed).  No page defines this
 * call; it is the host side of the library's bounded-wait error handling.
 */
fa_status fa_check_device_error(void* stream);

/*
 * Self-test of the timeout path: launches one warp that waits, with the
 * library's bounded wait, on a barrier nothing arrives on.  About one second
 * later it records FA_ERR_TIMEOUT in the device error word and exits normally
 * (no fault; the context stays usable), so fa_check_device_error(stream)
 * afterwards returns FA_ERR_TIMEOUT and clears the word.  For tests of callers'
 * error handling; the pages have no counterpart.
 */
fa_status fa_selftest_timeout(void* stream);

/* Number of kernel launches issued by this process through the library so
 * far (for checking that the native path ran).  No page defines this call. */
uint64_t fa_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_TILED_ATTENTION_FA_H */

/*
 * fa.h -- C ABI of libfa.so: exact IO-aware attention on NVIDIA B200
 * (sm_100a).  Forward writes O and the per-row log-sum-exp; backward
 * recomputes S and P from Q, K, V and that LSE and returns dQ, dK, dV.
 * No N x N score or probability matrix is ever written to device memory.
 *
 * What is computed ("注意力机制基础", section 2.1; "FlashAttention优化",
 * sections 3.1-3.2; "FlashAttention: Fast and Memory-Efficient Exact
 * Attention with IO-Awareness" review, 方法 items 1-3):
 *     S   = scale * Q K^T, with key j > query i set to -inf when causal
 *     P   = row softmax(S),  O = P V,  LSE_i = ln(sum_j exp(S_ij))
 * computed tile by tile with the online-softmax running max and sum.  The
 * backward is the derivative of the same definition:
 *     dV = P^T dO,  dP = dO V^T,  D_i = sum_k dO_ik O_ik,
 *     dS = P o (dP - D),  dQ = scale dS K,  dK = scale dS^T Q.
 *
 * Common argument conventions
 *   q, o, dO, dq : bf16, dense [B][N][Hq][d] or varlen [total][Hq][d]
 *   k, v, dk, dv : bf16, dense [B][N][Hkv][d] or varlen [total][Hkv][d]
 *                  (d contiguous; rows of one token are Hq*d or Hkv*d apart)
 *   lse          : fp32, dense [B][Hq][N] or varlen [Hq][total]; natural
 *                  log in the scaled-logit domain
 *   o_lo         : optional bf16 in q's layout (NULL: none): the forward's
 *                  second output, O - bf16(O) rounded to bf16, which the
 *                  backward adds to o when it forms D = rowsum(dO o O)
 *   B            : batch size; with cu_seqlens, the number of sequences
 *   Hq, Hkv      : query / key-value heads; Hq % Hkv == 0.  Query head h
 *                  reads key/value head h / (Hq / Hkv) (grouped-query
 *                  attention, "FlashAttention优化" section 5.3, read as
 *                  contiguous groups)
 *   N            : sequence length; with cu_seqlens, an upper bound on the
 *                  longest sequence (sizes the grid; no device->host read)
 *   d            : head dimension, 64 or 128
 *   scale        : multiplies Q K^T (normally 1/sqrt(d)), must be > 0
 *   causal       : nonzero -> key j is masked for query i when j > i
 *                  (positions counted from the start of each sequence)
 *   cu_seqlens   : NULL for dense inputs, else device int32[B+1] prefix sums
 *                  of the sequence lengths (padding-free batches).  The
 *                  kernels clamp every range they read from it to
 *                  [0, total_tokens], so a corrupt array (not starting at 0,
 *                  decreasing, past total_tokens, a length above N) gives
 *                  undefined results but no access outside the caller's
 *                  buffers; fa_validate_cu_seqlens() reports such an array
 *   total_tokens : with cu_seqlens, cu_seqlens[B] (the caller's allocation
 *                  size); ignored for dense inputs
 *   stream       : CUDA stream the kernels are enqueued on
 *
 * Ownership: the caller allocates every buffer (inputs, outputs, and the
 * backward workspace).  The library allocates no device memory at call time
 * and never synchronises the stream.  Its only device-resident state is the
 * error word below and one exception, described at fa_bwd_noalloc(): a fixed
 * FA_BWD_NOALLOC_SCRATCH_BYTES array that every GPU loading the library
 * holds until exit, whose device address is cached per device and whose
 * contents persist from call to call (overlapping fa_bwd_noalloc calls race
 * on it).  Host-side state is limited to settings (wait limit, profiling
 * events), cached driver entry points and that per-device address.  All
 * pointers are device pointers on one device and must be 16-byte aligned
 * (a NULL optional pointer included).  The kernels
 * run on the device that owns q: if it is not the calling thread's current
 * device, the call makes it current (this also gives a thread that has not
 * used CUDA before a context).  A host pointer for q is FA_ERR_INVALID_ARG.
 *
 * Errors: argument checks run on the host before any launch and return a
 * status without touching the device.  A launch failure returns
 * FA_ERR_CUDA.  Every wait inside the kernels is bounded; a wait that gives
 * up records a nonzero code that fa_device_error() reports once the caller
 * has synchronised the stream (the outputs are then undefined).
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad sizes, Hq % Hkv != 0 */
  FA_ERR_UNSUPPORTED = 2, /* d not in {64, 128} */
  FA_ERR_WORKSPACE = 3,   /* backward workspace missing or too small */
  FA_ERR_CUDA = 4         /* a CUDA runtime/driver call or launch failed */
} fa_status;

/*
 * Forward: O = softmax(scale Q K^T + mask) V and LSE.
 * Outputs o (bf16, q's layout) and lse (fp32, layout above) are fully
 * written for every valid token row; nothing else is touched.  When o_lo is
 * not NULL it receives, for the same rows, the rounding residual of o (the
 * fp32 result minus its bf16 rounding, itself rounded to bf16); o + o_lo
 * then carries about 16 significant bits of O.  Pass it on to fa_bwd: its
 * D = rowsum(dO o O) is otherwise formed from bf16 O, whose rounding error
 * reaches dK through the term -scale P_ij D_i Q_i (large for query rows of
 * large norm).  o_lo must not alias o.
 * Cites: "注意力机制基础" 2.1 (definition), "FlashAttention优化" 3.1 (tiling),
 * 3.2.1 (online softmax statistics m and l), paper review 方法 items 1-2
 * (tiles stay on chip, output rescale by exp(m_old - m_new)).
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, void* o_lo,
                 int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                 const int* cu_seqlens, int total_tokens, cudaStream_t stream);

/*
 * Bytes of device workspace fa_bwd needs: the fp32 row vector
 * D = rowsum(dO o O), fp16 copies of Q, K, V and dO (the backward's products
 * run on fp16 operands, see fa_bwd), a few KB of scale bookkeeping, and the
 * fp32 dQ accumulator.  The K and V copies are sized for Hkv = Hq, so the
 * figure holds for every grouping.  For dense inputs pass total_tokens =
 * B * N.  Returns 0 for invalid sizes.
 */
size_t fa_bwd_workspace_size(int B, int Hq, int N, int d, int total_tokens);

/*
 * Backward by recomputation (paper review, 方法 item 3): P is rebuilt from
 * Q, K and the forward's LSE; no S or P was stored.  Inputs q, k, v, o, lse,
 * o_lo (optional, NULL if the forward did not write it), dO as produced
 * for / by fa_fwd with the same sizes; outputs dq (q's
 * layout), dk and dv (k's layout; summed over the query heads of each
 * group).  `workspace` is caller-owned device memory of at least
 * fa_bwd_workspace_size() bytes, 256-byte aligned; its contents on entry do
 * not matter.  dQ accumulates in fp32 by atomic addition, so its low bits
 * may differ between runs; dK and dV are deterministic.
 * Precision: the five products of the backward take fp16 operands -- copies
 * of Q, K, V and dO each scaled by a power of two that puts its largest
 * magnitude just below 2^14 (exact for every bf16 value in fp16's normal
 * range), and P and dS rounded to fp16 (dS with its own power-of-two scale
 * from the bound |dS| <= 2 d max|dO| max|V|) -- with fp32 accumulation; the
 * scales are undone exactly in the epilogues.  fp16's 11 significant bits
 * keep dV and dK within 2e-2 of the exact gradient where bf16 operands (8
 * bits) did not.  Four kernels run in order: a max-magnitude pass, the
 * preprocess (copies, D, zeroed accumulator), the main kernel, the dQ
 * conversion.
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* o_lo, const void* dO, void* dq, void* dk, void* dv,
                 void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int N, int d,
                 float scale, int causal, const int* cu_seqlens, int total_tokens,
                 cudaStream_t stream);

/*
 * Block-sparse attention: the same forward and backward with every (query,
 * key) pair removed whose 128 x 128 tile the block mask does not allow -- a
 * generalisation of causal tile skipping ("FlashAttention优化" 7.2; the
 * paper review's block-sparse variant); exact on the allowed entries, and
 * disallowed tiles are never computed.
 *   block_mask        : device bytes [*][*][nt][nt], nt = ceil(N / 128);
 *                       tile (qt, kt) of sequence b and key/value head hk is
 *                       allowed iff block_mask[b * mask_batch_stride +
 *                       hk * mask_head_stride + qt * nt + kt] != 0
 *   mask_*_stride     : in elements; 0 uses one mask for all sequences /
 *                       all key/value heads.  The query heads of a group
 *                       share their key/value head's mask.
 * With causal, tiles above the diagonal stay skipped whatever the mask
 * says.  A query row with no allowed key gets O = 0, LSE = -inf and dQ = 0.
 * Dense batches only (no cu_seqlens) and N <= 65536 (FA_ERR_UNSUPPORTED
 * otherwise); every other argument as for fa_fwd / fa_bwd, including the
 * workspace size (fa_bwd_workspace_size with total_tokens = B * N).
 */
fa_status fa_fwd_blockmask(const void* q, const void* k, const void* v, void* o, float* lse,
                           void* o_lo, int B, int Hq, int Hkv, int N, int d, float scale,
                           int causal, const unsigned char* block_mask, long mask_batch_stride,
                           long mask_head_stride, cudaStream_t stream);

fa_status fa_bwd_blockmask(const void* q, const void* k, const void* v, const void* o,
                           const float* lse, const void* o_lo, const void* dO, void* dq,
                           void* dk, void* dv, void* workspace, size_t workspace_bytes, int B,
                           int Hq, int Hkv, int N, int d, float scale, int causal,
                           const unsigned char* block_mask, long mask_batch_stride,
                           long mask_head_stride, cudaStream_t stream);

/*
 * Capacity, in bytes, of the fixed scratch array behind fa_bwd_noalloc().
 */
#define FA_BWD_NOALLOC_SCRATCH_BYTES (64u << 20)

/*
 * Backward without any allocation -- an addition of this library; the pages
 * have no counterpart.  Same arguments, layouts and results as fa_bwd(),
 * minus the workspace: the scratch lives in one fixed 64 MiB array of
 * device memory inside the library (FA_BWD_NOALLOC_SCRATCH_BYTES), which
 * every GPU that loads the library holds until the process exits.
 *
 * For callers that cannot allocate device memory at call time -- for
 * example code running under a memory pool or allocator it must not
 * bypass, a runtime that forbids cudaMalloc/cudaFree on the hot path, or a
 * host that has no allocator of its own to hand the library.  This entry
 * point calls no cudaMalloc, cudaFree or allocating library routine.
 *
 * Limits and behaviour:
 *  - If the problem needs more scratch than the fixed capacity (compare
 *    fa_bwd_workspace_size() with FA_BWD_NOALLOC_SCRATCH_BYTES), the call
 *    returns FA_ERR_WORKSPACE before launching anything.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current and caches it; make
 *    that first call before any stream capture.
 *  - Every call on a device shares the one array, which keeps the last
 *    call's contents; each call re-initialises what it needs.  Calls whose
 *    kernels overlap on the GPU (different streams, no ordering between
 *    them) race on the array and give wrong results: serialise them.
 */
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* o_lo, const void* dO, void* dq, void* dk,
                         void* dv, int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                         const int* cu_seqlens, int total_tokens, cudaStream_t stream);

/*
 * Decode attention over a KV cache: one new query token per sequence
 * attends to the first L_b cached keys and values of its sequence
 * ("注意力机制基础" 2.3.1: autoregressive decoding re-reads the whole cache
 * for every token; "FlashAttention优化" 4.2).  For each sequence b and
 * query head h (key/value head h / (Hq / Hkv)):
 *     o[b][h]   = sum_j softmax_j(scale q[b][h] . k[b][j]) v[b][j],  j < L_b
 *     lse[b][h] = ln sum_j exp(scale q[b][h] . k[b][j])
 *   q, o             : bf16 [B][Hq][d]
 *   k_cache, v_cache : bf16 [B][Lmax][Hkv][d] (the training layout with
 *                      N = Lmax); rows at or past L_b are never used, so they
 *                      may hold anything
 *   lse              : fp32 [B][Hq]
 *   cache_seqlens    : device int32[B] with L_b (clamped to [0, Lmax]), or
 *                      NULL for L_b = Lmax.  A sequence with L_b = 0 gets
 *                      o = 0 and lse = -inf.
 *   workspace        : caller-owned device memory of at least
 *                      fa_decode_workspace_size() bytes, 256-byte aligned,
 *                      for the per-chunk partial results
 * The cache is cut into chunks processed in parallel and merged exactly
 * (lse = ln sum_s e^(lse_s), o = sum_s e^(lse_s - lse) o_s): a split
 * kernel and a merge kernel, after a one-block prefix kernel when
 * cache_seqlens is given.  The split and merge kernels are programmatic
 * dependent launches; each waits for the kernel before it on the stream
 * before touching memory, and the last one lets no later kernel start
 * early, so the call keeps ordinary stream order for the caller's work.  d must be 64
 * or 128 and Hq / Hkv at most 16 (FA_ERR_UNSUPPORTED otherwise); B and Hkv
 * at most 65535.  Same pointer, device, error and stream rules as fa_fwd.
 */
size_t fa_decode_workspace_size(int B, int Hq, int Lmax, int d);

fa_status fa_decode(const void* q, const void* k_cache, const void* v_cache, void* o,
                    float* lse, const int* cache_seqlens, int B, int Hq, int Hkv, int Lmax,
                    int d, float scale, void* workspace, size_t workspace_bytes,
                    cudaStream_t stream);

/*
 * Comparator only -- the softmax step of *standard* attention, which writes
 * the N x N probability matrix that fa_fwd never forms ("注意力机制基础"
 * 2.1 steps 2-3 and 2.2.2: S is read from and P written to device memory).
 * With S = Q K^T computed by a library GEMM per head, this reads
 *   s   : bf16 [BH][N][N], row i of head h at (h N + i) N (unscaled Q K^T)
 * and writes
 *   p   : bf16 [BH][N][N], P_ij = exp(scale S_ij - LSE_i) for allowed j, 0
 *         for j > i when causal
 *   lse : fp32 [BH][N], ln sum_j exp(scale S_ij) over the allowed j
 * so that O = P V is a second library GEMM.  One pass over HBM: 2 bytes
 * read and 2 written per element.  N must be a multiple of 8 and at most
 * 32768 (FA_ERR_UNSUPPORTED otherwise); BH * N must fit in an int; s and p
 * must not overlap.  Same pointer, device and error rules as fa_fwd.
 */
fa_status fa_std_softmax(const void* s, void* p, float* lse, int BH, int N, float scale,
                         int causal, cudaStream_t stream);

/*
 * Checks a cu_seqlens array on the device (one small kernel on `stream`,
 * reading cu_seqlens[0..B] only): cu[0] == 0, cu non-decreasing, every
 * length cu[b+1] - cu[b] at most N, and cu[B] <= total_tokens.  The first
 * failing rule (in that order) is recorded in the device error word as
 * 0x501, 0x502, 0x503 or 0x504, read by fa_device_error() after the caller
 * synchronises; nothing is recorded for a valid array.  The check is
 * optional: with the environment variable FA_DEBUG_VALIDATE set, every
 * varlen fa_fwd / fa_bwd call runs it first on its own stream.  No
 * counterpart on the pages; padding-free batches are the paper review's
 * "消除 padding".  Returns FA_ERR_INVALID_ARG for a NULL or misaligned
 * pointer or negative sizes, FA_ERR_CUDA if the launch fails.
 */
fa_status fa_validate_cu_seqlens(const int* cu_seqlens, int B, int N, int total_tokens,
                                 cudaStream_t stream);

/*
 * Device-side error word shared by all kernels of the library: 0 when no
 * wait has timed out (and no validation failed) since the last
 * fa_clear_device_error().  Reads device
 * memory synchronously on the current device; call after synchronising.
 * Returns -1 if the read itself fails.
 */
int fa_device_error(void);

/* Reset the device error word to 0 (synchronous). */
fa_status fa_clear_device_error(void);

/*
 * Limit, in nanoseconds, for every bounded wait inside the kernels launched
 * afterwards by this process (default 2e9 = 2 s).  Values below 1000 are
 * raised to 1000.  Host-side setting only; no device work.
 */
void fa_set_wait_limit_ns(unsigned long long ns);

/*
 * Diagnostic: launch one CTA that waits on an mbarrier nothing ever arrives
 * on, with the current wait limit, so that the bounded wait must give up.
 * It records its code in the error word and returns; the context stays
 * usable.  Used by the watchdog test.
 */
fa_status fa_watchdog_selftest(cudaStream_t stream);

/*
 * The cudaError_t value behind the most recent FA_ERR_CUDA returned to the
 * calling thread (0 if none).  Host-side, thread-local; no device work.
 */
int fa_last_cuda_error(void);

/*
 * Instrumentation: when main_begin / main_end are non-NULL, every later
 * fa_fwd / fa_bwd call made by this thread records them on its stream right
 * before and right after its main kernel (the attention kernel itself, not
 * the backward's pre- and post-processing kernels), so that the caller can
 * time that kernel with cudaEventElapsedTime.  Pass NULL, NULL to stop.  The
 * events stay owned by the caller.  Host-side setting only.
 */
void fa_set_profile_events(cudaEvent_t main_begin, cudaEvent_t main_end);

/* Human-readable name of a status code (static storage). */
const char* fa_status_string(fa_status s);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */

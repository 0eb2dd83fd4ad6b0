/*
 * fa.h -- C ABI of libfa: exact IO-aware scaled-dot-product attention for
 * NVIDIA B200 (sm_100a).
 *
 * The operation (hysenlabs "FlashAttention: GPU-specific backends and the
 * attention API", section on outputs and operations; Qiita Flash Attention
 * tutorial, section 2.2):
 *
 *     O = softmax(Q K^T * scale) V
 *
 * computed by tiling with an online softmax so that the N x N score and
 * probability matrices never reach device memory (Qiita tutorial, sections
 * 4.2-4.3; abeam.tech FlashAttention summary, "computing softmax blockwise
 * correctly" and "cutting memory traffic by tiling").  The forward pass also
 * writes the per-row log-sum-exp; the backward pass recomputes P from it
 * (abeam.tech summary, "backward uses recomputation").
 *
 * Tensor layout (row-major, last index contiguous, no padding):
 *     q, o, dO, dq : [B, Nq, Hq,  d]
 *     k, v, dk, dv : [B, Nk, Hkv, d]
 *     lse          : [B, Hq, Nq]      fp32, natural log, scale included:
 *                    lse[b,h,i] = ln sum_j exp(scale * q_i . k_j) over visible j
 * bf16 entry points take and return __nv_bfloat16 data (passed as void*);
 * the _f16 entry points the same with IEEE fp16 data; the _f32 entry points
 * take float data.  Accumulation is fp32 throughout.
 *
 * Masking (hysenlabs page, option list and changelog v2.1 / v2.3): with
 * delta = Nk - Nq, key j is visible to query i iff
 *     (wr < 0 || j <= i + delta + wr)  &&  (win_l < 0 || j >= i + delta - win_l)
 * where wr = 0 when causal != 0 and wr = win_r otherwise.  Bounds are
 * inclusive; a negative bound is unbounded.  The causal diagonal is aligned to
 * the bottom-right corner when Nq != Nk.  A query row with no visible key gets
 * O = 0, lse = -inf and zero gradients.
 *
 * MQA / GQA (hysenlabs page, option list): Hq must be divisible by Hkv; query
 * head h reads key/value head h / (Hq / Hkv).
 *
 * Ownership and execution: the caller allocates and owns every buffer (device
 * memory unless stated).  Calls are ordered on `stream` (a cudaStream_t; NULL is
 * the legacy default stream) and return without synchronising; the library
 * allocates no device memory.  All pointers must be device pointers aligned to
 * 16 bytes.  Argument errors are reported before anything is launched.  A
 * kernel that gives up on a bounded wait records FA_ERR_TIMEOUT in a
 * per-device status word that fa_get_device_status() reads.
 *
 * There is no CPU fallback: every entry point runs only its CUDA kernels.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fa_stream_t; /* same type as cudaStream_t */

enum fa_status {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, Hq % Hkv != 0, non-finite scale */
  FA_ERR_UNSUPPORTED = 2, /* head dim not in {64, 128, 256} (bf16) or > 256 (f32) */
  FA_ERR_CUDA = 3,        /* a CUDA runtime/driver call or launch failed */
  FA_ERR_WORKSPACE = 4,   /* workspace missing or smaller than fa_bwd_workspace_size() */
  FA_ERR_TIMEOUT = 5      /* a device-side bounded wait expired (see fa_get_device_status) */
};

/*
 * Forward pass, bf16 in / bf16 out, fp32 accumulation.
 *   q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d] : inputs (bf16, device)
 *   o [B,Nq,Hq,d]                   : output (bf16, device)
 *   lse [B,Hq,Nq]                   : output (fp32, device)
 *   d in {64, 128, 256}; scale is usually 1/sqrt(d).
 * Returns FA_OK or an fa_status code.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Nq,
           int Nk, int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r,
           fa_stream_t stream);

/*
 * Forward pass over packed variable-length sequences (hysenlabs changelog
 * v2.0: the varlen functions), bf16.  The B sequences are stored back to back:
 *   q, o [total_q, Hq, d], k, v [total_k, Hkv, d]  (bf16, device)
 *   lse [Hq, total_q]                                (fp32, device)
 *   cu_seqlens_q, cu_seqlens_k [B + 1]               (int32, device, 4-byte aligned)
 * Sequence b is query rows [cu_seqlens_q[b], cu_seqlens_q[b+1]) and key rows
 * [cu_seqlens_k[b], cu_seqlens_k[b+1]); it attends to its own keys only, with
 * fa_fwd's masks applied to its own lengths (causal bottom-right per
 * sequence).  The caller guarantees 0 <= cu[b] <= cu[b+1] <= total and every
 * length <= max_seqlen (a longer sequence is computed only up to
 * max_seqlen_q rows); the kernel never writes outside [0, total_q) rows of o
 * and lse whatever the offsets hold.  Rows of o and lse not covered by any
 * sequence are left untouched.  Other arguments as fa_fwd.
 */
int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int max_seqlen_q,
                  int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int d, float scale,
                  int causal, int win_l, int win_r, fa_stream_t stream);

/*
 * Bytes of device workspace fa_bwd needs for these sizes: two fp32 arrays
 * [B, Hq, Nq rounded up to 256], the row sums D = rowsum(dO * O) and the
 * saved LSE in base 2.  Returns 0 for invalid sizes.
 */
size_t fa_bwd_workspace_size(int B, int Nq, int Hq, int d);

/*
 * Backward pass, bf16, fp32 accumulation, deterministic (the same inputs give
 * the same bits on every call).
 *   q, k, v, o, lse : the forward's inputs and outputs
 *   dO [B,Nq,Hq,d]  : gradient of the loss with respect to o (bf16)
 *   dq [B,Nq,Hq,d], dk/dv [B,Nk,Hkv,d] : outputs (bf16); dk and dv are summed
 *                     over the Hq/Hkv query heads that share a key/value head
 *   workspace       : device buffer of at least fa_bwd_workspace_size() bytes,
 *                     16-byte aligned, owned by the caller, contents ignored
 * Gradients are those of sum(dO * O) with respect to q, k and v, with P
 * recomputed from lse.  Returns FA_OK or an fa_status code.
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dO, void* dq, void* dk, void* dv, int B, int Nq, int Nk, int Hq, int Hkv,
           int d, float scale, int causal, int win_l, int win_r, void* workspace,
           size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_bwd without a workspace argument, for callers that cannot allocate
 * device memory: an allocator-free runtime (an inference engine that carves
 * all of its device memory out of one arena at start-up and forbids
 * cudaMalloc afterwards), a host program with a fixed memory budget that has
 * no cudaMalloc on its path, or code that records work into a CUDA graph and
 * must not allocate while doing so.  The pages have no counterpart; it is an
 * addition of this library.
 *
 * Same arguments, results and determinism as fa_bwd (the same kernels run, so
 * the outputs are bit-identical to fa_bwd's).  Its scratch (the bytes
 * fa_bwd_workspace_size() reports for these sizes) lives in a fixed 16 MiB
 * array inside the library's device image, which every GPU that loads the
 * library holds until the process exits; problems whose workspace would not
 * fit get FA_ERR_WORKSPACE, without anything being launched.  The library
 * calls no cudaMalloc/cudaFree and no allocating routine on this path.
 *
 * The first backward call on a device (this one or fa_bwd) sets up
 * per-device state: it looks up the array's device address
 * (cudaGetSymbolAddress) with that device current and sets the kernels'
 * shared-memory attributes; the first call from a given caller stream also
 * creates that stream's side stream and two events.  Make one eager call on
 * each device before any stream capture.  While the caller's stream is being
 * captured, the backward keeps all of its launches on that stream.  Every
 * call on a device shares the one array and overwrites it (the call clears
 * what must start at zero itself): calls that can overlap on the GPU -- on
 * different streams without ordering between them, or graph replays that
 * overlap another call -- race on it and must be serialised by the caller.
 */
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dO, void* dq, void* dk, void* dv, int B, int Nq, int Nk, int Hq,
                   int Hkv, int d, float scale, int causal, int win_l, int win_r,
                   fa_stream_t stream);

/*
 * Forward pass for few query rows against a long key/value sequence
 * (decoding with a KV cache; hysenlabs page, changelog v2.2), bf16, with the
 * arguments, masks, GQA mapping and outputs of fa_fwd: o and lse hold the same
 * attention result (up to fp32 summation order).  The key range is split
 * across CTAs, each CTA handling the Hq/Hkv query heads of one key/value head
 * together (K and V are read from HBM once per key/value head, not once per
 * query head).  One kernel launch: the last CTA of each (batch, key/value
 * head, query tile) to finish merges the splits' partial outputs through
 * their log-sum-exp, in split order, so results are deterministic.
 *   n_splits : key splits per (batch, key/value head, query tile); 0 lets the
 *              library choose from the current device's SM count (the same
 *              choice fa_fwd_splitkv_workspace_size makes with that device
 *              current); at most 4096
 *   workspace: device buffer of at least fa_fwd_splitkv_workspace_size() bytes,
 *              16-byte aligned, owned by the caller, contents ignored (each
 *              call tags the per-unit counters it keeps there and leaves them
 *              at zero; CUDA graph replays are fine); may be NULL when that
 *              size is 0 (no split).  Calls that can overlap on the GPU must
 *              not share a workspace.
 * Requires Hq / Hkv <= 128 (else FA_ERR_UNSUPPORTED) and d in {64, 128, 256}.
 * Any Nq is accepted; query rows are packed into 128-row tiles of
 * floor(128 / (Hq/Hkv)) queries, so it pays off while Nq * Hq / Hkv is small.
 * Returns FA_OK or an fa_status code (FA_ERR_WORKSPACE: workspace missing or
 * too small).
 */
size_t fa_fwd_splitkv_workspace_size(int B, int Nq, int Nk, int Hq, int Hkv, int d, int causal,
                                     int win_l, int win_r, int n_splits);
int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Nq,
                   int Nk, int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r,
                   int n_splits, void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_fwd_splitkv over a key/value cache, with the cache update of
 * hysenlabs' `flash_attn_with_kvcache` (Python-interface section): the new
 * keys and values are written into the caches in place, then the query rows
 * attend to each sequence's cached keys plus the new ones.
 *   k_cache, v_cache [B, Nk, Hkv, d] : caches (bf16, device); Nk is their
 *                      capacity in keys.  Updated in place when n_new > 0.
 *   k_new, v_new [B, n_new, Hkv, d]   : keys/values to append (bf16, device);
 *                      ignored (may be NULL) when n_new == 0
 *   cache_seqlens [B] : int32, device, 4-byte aligned: keys already cached
 *                      per sequence.  Row t of k_new/v_new goes to cache row
 *                      cache_seqlens[b] + t (rows at or past Nk are dropped),
 *                      and sequence b attends to its first
 *                      min(Nk, cache_seqlens[b] + n_new) keys.  NULL: every
 *                      sequence holds all Nk keys (then n_new must be 0).
 *                      The array is not modified.
 *   q, o, lse, masks, n_splits, workspace: as fa_fwd_splitkv, with the
 *                      workspace size from fa_fwd_kvcache_workspace_size.
 *                      The causal diagonal and the window of sequence b are
 *                      aligned to its own key count (bottom-right).
 * The keys are split in chunks of equal length planned for the full capacity
 * Nk, so a shorter sequence takes fewer CTAs.  With cache_seqlens given and
 * n_splits 0, the library plans about three waves of CTAs at full length
 * (instead of one), so that ragged batches balance.
 * Returns FA_OK or an fa_status code.
 */
size_t fa_fwd_kvcache_workspace_size(int B, int Nq, int Nk, int Hq, int Hkv, int d, int causal,
                                     int win_l, int win_r, int n_splits, int with_seqlens);
int fa_fwd_kvcache(const void* q, void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                   const int* cache_seqlens, void* o, float* lse, int B, int Nq, int Nk, int n_new,
                   int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r, int n_splits,
                   void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * Backward pass over packed variable-length sequences: the gradients of
 * fa_fwd_varlen, in its layouts (dq like q [total_q, Hq, d], dk / dv like k
 * [total_k, Hkv, d]; o, lse and dO as fa_fwd_varlen wrote / received them),
 * deterministic, with fa_bwd's arguments otherwise.  The workspace holds the
 * row statistics per sequence padded to max_seqlen_q: at least
 * fa_bwd_workspace_size(B, max_seqlen_q, Hq, d) bytes.  Rows of dq, dk and dv
 * not covered by any sequence are left untouched.  The caller guarantees the
 * offsets as for fa_fwd_varlen; the kernels never write outside
 * [0, total) rows whatever they hold.
 */
int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                  const void* dO, void* dq, void* dk, void* dv, const int* cu_seqlens_q,
                  const int* cu_seqlens_k, int B, int max_seqlen_q, int max_seqlen_k, int total_q,
                  int total_k, int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r,
                  void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * Block-sparse forward (abeam.tech FlashAttention summary, the block-sparse
 * extension): fa_fwd with the 128 x 128 (query block, key block) tiles that
 * block_mask marks zero left out -- their keys are invisible to their query
 * rows, on top of the causal / window masks -- and the kernel skips them.
 *   block_mask : uint8, device; for batch b and query head h the mask is
 *                block_mask + b * mask_stride_b + h * mask_stride_h, a
 *                row-major [ceil(Nq / 128)][ceil(Nk / 128)] array, nonzero =
 *                computed.  Strides are in bytes (elements); 0 shares one
 *                mask across batches or heads.
 * Rows that see no key (every block of their row off) get O = 0 and
 * LSE = -inf.  FA_ERR_UNSUPPORTED also when Nk needs more than the shared
 * memory left for the CTA's key-tile list (Nk in the hundreds of
 * thousands).  fa_fwd_blocksparse_f16 takes fp16 tensors.
 */
int fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse,
                       const unsigned char* block_mask, long long mask_stride_b, long long mask_stride_h,
                       int B, int Nq, int Nk, int Hq, int Hkv, int d, float scale, int causal, int win_l,
                       int win_r, fa_stream_t stream);
int fa_fwd_blocksparse_f16(const void* q, const void* k, const void* v, void* o, float* lse,
                           const unsigned char* block_mask, long long mask_stride_b, long long mask_stride_h,
                           int B, int Nq, int Nk, int Hq, int Hkv, int d, float scale, int causal, int win_l,
                           int win_r, fa_stream_t stream);

/*
 * Block-sparse backward: the gradients of fa_fwd_blocksparse with the same
 * block mask (the skipped tiles contribute nothing, and are not computed),
 * deterministic, with fa_bwd's other arguments and workspace.
 * FA_ERR_UNSUPPORTED also when the per-CTA lists of tiles do not fit in
 * shared memory (Nk or (Hq / Hkv) * Nq in the hundreds of thousands).
 */
int fa_bwd_blocksparse(const void* q, const void* k, const void* v, const void* o, const float* lse,
                       const void* dO, void* dq, void* dk, void* dv, const unsigned char* block_mask,
                       long long mask_stride_b, long long mask_stride_h, int B, int Nq, int Nk, int Hq,
                       int Hkv, int d, float scale, int causal, int win_l, int win_r, void* workspace,
                       size_t workspace_bytes, fa_stream_t stream);
int fa_bwd_blocksparse_f16(const void* q, const void* k, const void* v, const void* o, const float* lse,
                           const void* dO, void* dq, void* dk, void* dv, const unsigned char* block_mask,
                           long long mask_stride_b, long long mask_stride_h, int B, int Nq, int Nk, int Hq,
                           int Hkv, int d, float scale, int causal, int win_l, int win_r, void* workspace,
                           size_t workspace_bytes, fa_stream_t stream);

/*
 * fp16 variants (hysenlabs page, requirements: fp16 and bf16 inputs): the
 * same arguments, semantics, layouts and workspace sizes as the bf16 entry
 * points of the same name without the suffix, with every 16-bit tensor
 * (q, k, v, o, dO, dq, dk, dv, k_new, v_new, the caches) holding IEEE fp16
 * instead of bf16.  Accumulation stays fp32; P and dS enter the tensor cores
 * as fp16 (P <= 2^8 in the forward, P <= 1 in the backward, within range).
 */
int fa_fwd_f16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Nq,
               int Nk, int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r,
               fa_stream_t stream);
int fa_bwd_f16(const void* q, const void* k, const void* v, const void* o, const float* lse,
               const void* dO, void* dq, void* dk, void* dv, int B, int Nq, int Nk, int Hq, int Hkv,
               int d, float scale, int causal, int win_l, int win_r, void* workspace,
               size_t workspace_bytes, fa_stream_t stream);
int fa_fwd_varlen_f16(const void* q, const void* k, const void* v, void* o, float* lse,
                      const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int max_seqlen_q,
                      int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int d, float scale,
                      int causal, int win_l, int win_r, fa_stream_t stream);
int fa_bwd_varlen_f16(const void* q, const void* k, const void* v, const void* o, const float* lse,
                      const void* dO, void* dq, void* dk, void* dv, const int* cu_seqlens_q,
                      const int* cu_seqlens_k, int B, int max_seqlen_q, int max_seqlen_k, int total_q,
                      int total_k, int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r,
                      void* workspace, size_t workspace_bytes, fa_stream_t stream);
int fa_fwd_splitkv_f16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Nq,
                       int Nk, int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r,
                       int n_splits, void* workspace, size_t workspace_bytes, fa_stream_t stream);
int fa_fwd_kvcache_f16(const void* q, void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                       const int* cache_seqlens, void* o, float* lse, int B, int Nq, int Nk, int n_new,
                       int Hq, int Hkv, int d, float scale, int causal, int win_l, int win_r, int n_splits,
                       void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * fp32 variants for small problems (fp32 in, fp32 out, fp32 arithmetic on the
 * CUDA cores).  Same arguments and semantics as fa_fwd / fa_bwd; d <= 256 and
 * d a multiple of 32.
 */
int fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B,
               int Nq, int Nk, int Hq, int Hkv, int d, float scale, int causal, int win_l,
               int win_r, fa_stream_t stream);
int fa_bwd_f32(const float* q, const float* k, const float* v, const float* o, const float* lse,
               const float* dO, float* dq, float* dk, float* dv, int B, int Nq, int Nk, int Hq,
               int Hkv, int d, float scale, int causal, int win_l, int win_r, void* workspace,
               size_t workspace_bytes, fa_stream_t stream);

/*
 * Ring (context-parallel) attention: combining partial results.  A long
 * sequence is split across GPUs; each GPU keeps its slice of query rows while
 * the key/value slices travel around the ring of GPUs (zocula.com fla guide,
 * the flame bullets and the glossary entry on context parallelism).  Each GPU
 * runs fa_fwd / fa_bwd on its (query slice, key/value slice) pairs; these two
 * calls combine the pieces.
 *
 * fa_lse_merge folds the forward result over one more key set into a
 * running result (abeam.tech FlashAttention summary, "computing softmax
 * blockwise correctly", applied to whole key sets): with lse_s the natural
 * log-sum-exp and O_s the normalised output of set s,
 *     lse = ln sum_s exp(lse_s),   O = sum_s exp(lse_s - lse) O_s.
 *   o_acc  [B, Nq_acc, H, d] fp32, lse_acc [B, H, Nq_acc] fp32 : the running
 *            result, updated in place on rows [row0, row0 + Nq); with
 *            first != 0 those rows are overwritten by the part (their
 *            contents are ignored)
 *   o_part [B, Nq, H, d] bf16 (_f16: fp16), lse_part [B, H, Nq] fp32 : the
 *            result of rows row0 .. row0 + Nq - 1 over the next key set, as
 *            fa_fwd wrote it
 *   o_out  [B, Nq_acc, H, d] bf16 / fp16, or NULL: the merged O of rows
 *            [row0, row0 + Nq), rounded (other rows untouched)
 *   d in {64, 128, 256}; 0 <= row0, row0 + Nq <= Nq_acc (Nq_acc = Nq,
 *   row0 = 0 when the part covers every row).  Rows empty in both
 *   (lse = -inf) stay O = 0, lse = -inf.  Merging parts in a fixed order
 *   gives the same bits every time.
 *
 * fa_grad_accumulate sums backward shares in fp32: the gradients fa_bwd
 * computes for one key set, given the full rows' o and lse, are that set's
 * share of dq and its keys' dk / dv.  Tensors are B batches of rows of
 * row_elems elements (a row: all heads of one sequence position, H * d);
 * the part covers rows [row0, row0 + rows) of the accumulator.
 *   acc  [B, rows_acc, row_elems] fp32 : running sum, updated in place on
 *          rows [row0, row0 + rows) (first != 0: those rows = part)
 *   part [B, rows, row_elems] bf16 / fp16, or NULL (only convert)
 *   out  [B, rows_acc, row_elems] bf16 / fp16, or NULL: the sum, rounded,
 *          written on the same rows
 *   1 <= B <= 65535, 0 <= row0, row0 + rows <= rows_acc, row_elems a
 *   multiple of 8; at least one of part, out given.  A flat sum of n
 *   elements is B = rows_acc = rows = 1, row0 = 0, row_elems = n.
 * Both return FA_OK or FA_ERR_INVALID_ARG / FA_ERR_UNSUPPORTED / FA_ERR_CUDA;
 * pointers are device pointers aligned to 16 bytes; stream-ordered.
 */
int fa_lse_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, void* o_out, int B,
                 int Nq, int H, int d, int Nq_acc, int row0, int first, fa_stream_t stream);
int fa_lse_merge_f16(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, void* o_out, int B,
                     int Nq, int H, int d, int Nq_acc, int row0, int first, fa_stream_t stream);
int fa_grad_accumulate(float* acc, const void* part, void* out, int B, int rows_acc, int row0, int rows,
                       long long row_elems, int first, fa_stream_t stream);
int fa_grad_accumulate_f16(float* acc, const void* part, void* out, int B, int rows_acc, int row0, int rows,
                           long long row_elems, int first, fa_stream_t stream);

/*
 * Synchronises `stream`, then returns and clears the device status word of
 * the current device: FA_OK, FA_ERR_TIMEOUT if a kernel gave up on a bounded
 * wait since the last call, or FA_ERR_CUDA if the synchronisation failed.
 */
int fa_get_device_status(fa_stream_t stream);

/*
 * Test only (failure detection): arms a one-shot for the next dense fa_fwd /
 * fa_fwd_f16 launch in this process, in which the producer of the first CTA
 * issues no key/value load after its first ring stages.  That CTA's MMA
 * thread then waits for a copy that never comes; its bounded wait (2 s) runs
 * out, the CTA raises the device status word, waits for the copies it did
 * issue and frees its tensor memory, and the launch ends normally with that
 * CTA's output rows unwritten.  fa_get_device_status then returns
 * FA_ERR_TIMEOUT; the context stays usable.  Nothing is faulted, trapped or
 * hung.  Returns FA_OK.
 */
int fa_test_withhold_next_load(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* fa_status_string(int status);

/*
 * Kernel tracing.  While enabled, every kernel the library launches is
 * bracketed by two CUDA events recorded on the stream it runs on (the
 * caller's, or for the backward's dQ kernel the library's side stream of the
 * device, forked from and joined back into the caller's stream) (events come
 * from a pool created when tracing is switched on; no device memory is
 * allocated).  fa_trace_read() waits for the recorded events, adds each
 * launch's device time to ms[kind] and one to launches[kind] for the
 * FA_KERNEL_KINDS kinds below (both arrays are caller-owned host memory of
 * FA_KERNEL_KINDS entries, zeroed by the library), then forgets the records.
 * Returns FA_OK, FA_ERR_INVALID_ARG (null array) or FA_ERR_CUDA.
 */
enum fa_kernel_kind {
  FA_KERNEL_FWD = 0,      /* forward, bf16 (tcgen05) */
  FA_KERNEL_BWD_PREP = 1, /* backward preprocess D = rowsum(dO * O) */
  FA_KERNEL_BWD_DQ = 2,   /* backward dQ, bf16 (tcgen05) */
  FA_KERNEL_BWD_DKDV = 3, /* backward dK/dV, bf16 (tcgen05) */
  FA_KERNEL_F32 = 4,      /* any fp32-path kernel */
  FA_KERNEL_DECODE = 5,   /* fa_fwd_splitkv / fa_fwd_kvcache, bf16 (tcgen05) */
  FA_KERNEL_KVCACHE_APPEND = 6, /* fa_fwd_kvcache: new keys/values into the cache */
  FA_KERNEL_BWD_CALL = 7, /* not a kernel: a whole backward call, preprocess to the end of
                             the dQ and dK/dV kernels (which run concurrently) */
  FA_KERNEL_MERGE = 8,    /* fa_lse_merge / fa_grad_accumulate */
  FA_KERNEL_KINDS = 9
};
int fa_trace_enable(int on);
int fa_trace_read(double* ms, long long* launches);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */

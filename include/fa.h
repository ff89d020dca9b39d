/*
 * fa.h - C ABI of the B200 (sm_100a) exact-attention library (libfa.so).
 *
 * The library computes exact scaled-dot-product attention,
 *     O = softmax(scale * Q K^T [+ causal mask]) V,
 * the definition printed on every page it follows (e.g. the opening formula of
 * "Flash-Attention 2/3在ms-swift中的集成与性能提升" and section 一 of the Qwen
 * flash_attn explainer), computed tile by tile with a running row max and row sum
 * ("FlashAttention优化Transformer显存与计算效率", sections 2.2.1-2.2.3) so the N x N
 * score matrix never reaches global memory.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are DEVICE pointers to contiguous row-major arrays. Q, K, V, O and their
 *    gradients are bf16 (passed as void*, 2 bytes per element) in the layout
 *    [B, N, H, d] = (batch, seq_len, heads, head_dim), the layout of section 1.1 of
 *    "ms-swift长文本训练优化，Flash-Attention显存省一半". Every bf16 pointer must be
 *    16-byte aligned; float pointers 4-byte aligned. (fa_fwd_ex / fa_bwd_ex also take
 *    row strides and packed variable-length batches, fa_decode_paged a paged cache;
 *    their comments give the layouts.)
 *  - d (head_dim) must be 64 or 128. The device must be compute capability 10.0
 *    (B200, sm_100a).
 *  - scale is the softmax scale; any finite value. (The pages' softmax_scale=None
 *    default, 1/sqrt(d), is applied by the Python binding, not here.)
 *  - LSE is the natural-log log-sum-exp of each query row's scaled scores over its
 *    visible keys, fp32, laid out [B, H, N] ([H, total] for a packed variable-length
 *    call). A row with no visible key gets -inf.
 *  - causal != 0 masks key j for query i when j > i (for decode, the single new
 *    query sees every valid key, so causal changes nothing there).
 *  - stream is a cudaStream_t (NULL = legacy default stream). Every call only
 *    enqueues work on that stream and returns without synchronising.
 *  - Ownership: the caller allocates and owns every buffer, including workspaces;
 *    the library allocates no device memory and keeps no per-call state. Inputs are
 *    read-only except the KV cache rows that fa_decode appends.
 *  - Work scheduling: the forward and backward kernels are persistent (one CTA per
 *    SM, each taking work units from a counter). The backward's counter lives in the
 *    caller's workspace. The forward's comes from a pool of 64 counters in the
 *    library's device image, one per launch in turn, zeroed on the launch's stream;
 *    so at most 64 forward launches may be executing at the same time on one device
 *    (more, on many streams with no ordering between them, could share a counter).
 *  - Errors: argument problems are detected on the host before anything is
 *    launched and return a non-zero status with a message from fa_last_error().
 *    Problems only visible on the device (a cache_seqlens value out of range, an
 *    internal pipeline wait that timed out) are recorded in a device status word
 *    and read back by fa_device_status().
 *  - Empty problems (B, N or H equal to 0) return FA_OK without launching.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment, non-finite scale */
  FA_ERR_UNSUPPORTED = 2,   /* d not in {64,128}, or device is not sm_100 */
  FA_ERR_CUDA = 3,          /* a CUDA runtime/driver call or kernel launch failed */
  FA_ERR_WORKSPACE = 4,     /* workspace pointer null or smaller than required */
  FA_ERR_TIMEOUT = 5,       /* (device) a pipeline wait gave up; results are invalid */
  FA_ERR_DEVICE_INPUT = 6   /* (device) cache_seqlens out of range / cache full */
} fa_status;

/*
 * Fused forward: out = softmax(scale*Q K^T, mask) V and lse, in one kernel.
 *   q, k, v : [B, N, H, d] bf16 (read)        out : [B, N, H, d] bf16 (written)
 *   lse     : [B, H, N] fp32 (written)
 * Follows the forward pass of the pages: tiling + blockwise softmax + fusion
 * ("FlashAttention优化Transformer显存与计算效率" 2.2), fp32 softmax accumulation with
 * bf16 in/out (same page 3.2), causal flag (flash_attn_func(..., causal=True)).
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                 int B, int H, int N, int d, int causal, float scale, void* stream);

/*
 * Extended forward: the computation of fa_fwd with three generalisations.
 *  - Row strides (packed QKV). Every row-major operand may have consecutive tokens
 *    *_row_stride elements apart (a multiple of 8, at least H*d), so q, k and v can
 *    be views into one packed [B, N, 3, H, d] tensor (q = base, k = base + H*d,
 *    v = base + 2*H*d, row stride 3*H*d), the layout of flash_attn_qkvpacked_func in
 *    "突破AI算力瓶颈：FlashAttention与MindSpore 2.0全场景融合方案" (核心API与使用示例).
 *    Contiguous tensors have row stride H*d.
 *  - Variable-length batches (packing, "ms-swift长文本训练优化，Flash-Attention显存省一半"
 *    sections 4.2 and 5.1, flash_attn_varlen_func in section 4.3). With cu_seqlens
 *    NULL the layout is the dense [B, N, H, d] (row (b, n) is token b*N + n) and lse
 *    is [B, H, N]. With cu_seqlens (DEVICE int32 [B + 1], non-decreasing, cu[0] = 0,
 *    cu[B] = total_tokens) the operands are [total_tokens, H, d], sequence b is
 *    tokens [cu[b], cu[b+1]), N is an upper bound on every sequence length (it sizes
 *    the grid), lse is [H, total_tokens], and attention never crosses sequences.
 *    Entries that break these rules are reported as FA_ERR_DEVICE_INPUT through
 *    fa_device_status and the affected sequences are left unwritten.
 *    A tile that runs past the end of a sequence reads the next sequence's rows and
 *    gives them probability 0: those rows must hold finite values (any finite values).
 *  - Sliding window ("Flash-Attention 2/3在ms-swift中的集成与性能提升", FA3 feature
 *    list: structured masks such as the sliding window). Query i sees keys
 *    [i - window_left, i + window_right] within its sequence; -1 leaves that side
 *    unbounded. causal != 0 is window_right = 0 (window_right must then be 0 or -1).
 *    Key tiles outside every row's window are skipped, not masked.
 * Errors as fa_fwd; a bad stride or window edge is FA_ERR_INVALID_ARG.
 */
fa_status fa_fwd_ex(const void* q, const void* k, const void* v, void* out, float* lse,
                    const int* cu_seqlens, int total_tokens, int B, int H, int N, int d,
                    long long q_row_stride, long long k_row_stride, long long v_row_stride,
                    long long out_row_stride, int causal, int window_left, int window_right,
                    float scale, void* stream);

/* Bytes of device workspace fa_bwd needs for these sizes (fp32 dQ accumulator, the
 * per-row D = rowsum(dO * O) and LSE vectors, and the work-unit counter of the
 * persistent kernel). Pure function of its arguments. */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward with recomputation: from q, k, v, out, dout and the forward's lse,
 * rebuild P = exp(scale*Q K^T - lse) tile by tile (the score matrix is recomputed,
 * not stored, as the pages' "重计算 / Recomputation" item describes) and write
 *   dv = P^T dO,  dk = scale * dS^T Q,  dq = scale * dS K,
 *   where dS = P * (dO V^T - D),  D_i = sum_c dO_ic O_ic.
 *   q, k, v, out, dout : [B, N, H, d] bf16 (read);  lse : [B, H, N] fp32 (read)
 *   dq, dk, dv         : [B, N, H, d] bf16 (written)
 *   workspace          : >= fa_bwd_workspace_size(B,H,N,d) bytes, 256-byte aligned;
 *                        contents on entry are ignored and left undefined. It holds the
 *                        call's dQ accumulator and work-unit counter, so two calls whose
 *                        executions may overlap (different streams, no ordering) need
 *                        separate workspaces.
 * dq is summed over key tiles with fp32 reductions into the workspace in an order
 * that is not fixed, so dq may differ in the last bits between runs; dk and dv are
 * bitwise repeatable (fa_bwd_ex with deterministic = 1 makes dq repeatable too).
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
                 const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                 int causal, float scale, void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_bwd with the same arguments, plus two optional CUDA events (cudaEvent_t, either
 * may be NULL) that are recorded on `stream` immediately before and immediately after
 * the main backward kernel (the one that recomputes P and runs the five tile
 * products). A caller can then time that kernel alone with cudaEventElapsedTime
 * while the whole backward still runs as one call. Events are not created,
 * synchronised or destroyed by the library.
 */
fa_status fa_bwd_profiled(const void* q, const void* k, const void* v, const void* out,
                          const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                          int H, int N, int d, int causal, float scale, void* workspace,
                          size_t workspace_bytes, void* stream, void* main_start,
                          void* main_stop);

/*
 * Extended backward: the gradients of fa_fwd_ex, with the same row strides,
 * variable-length batches and sliding window (see fa_fwd_ex). row_strides is a HOST
 * array of 8 strides in elements, for q, k, v, out, dout, dq, dk, dv in that order
 * (so dq, dk, dv can be views into one packed [B, N, 3, H, d] gradient). lse is the
 * forward's ([B, H, N] dense, [H, total_tokens] variable length). The workspace is
 * fa_bwd_workspace_size(B, H, N, d) bytes with N the largest sequence length.
 * deterministic: 0 runs the fused backward of fa_bwd (dq summed over key tiles with
 * fp32 reductions whose order is not fixed); nonzero runs two kernels instead, one
 * per key tile writing dk and dv and one per query tile writing dq, each gradient
 * element written once, so all three gradients are bitwise repeatable on the same
 * inputs (the flash_attn `deterministic` flag of the MindSpore page, section
 * 常见问题与解决方案). That path recomputes the scores twice (seven tile products per
 * tile pair instead of five) and is slower. Errors as fa_bwd and fa_fwd_ex.
 */
fa_status fa_bwd_ex(const void* q, const void* k, const void* v, const void* out, const void* dout,
                    const float* lse, void* dq, void* dk, void* dv, const int* cu_seqlens,
                    int total_tokens, int B, int H, int N, int d, const long long* row_strides,
                    int causal, int window_left, int window_right, float scale, int deterministic,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_bwd for callers that cannot allocate device memory. Some callers have no way
 * to hand this library a workspace: a host runtime that reserved all device memory
 * at start-up and refuses later allocations, plugin or interpreter code that has
 * no access to the application's allocator, or a latency-critical loop that must
 * not call an allocator (which may synchronise the device). This entry point takes
 * the same inputs and outputs as fa_bwd, minus the workspace, and uses a scratch
 * array that lives inside the library instead. The FlashAttention pages have no counterpart to
 * this call; it only exists for such callers.
 *
 * Limits and behaviour:
 *  - The scratch is a fixed 32 MiB array (FA_BWD_NOALLOC_SCRATCH_BYTES) that every
 *    GPU holds for as long as the library is loaded. Problems whose workspace
 *    (fa_bwd_workspace_size) exceeds it are rejected with FA_ERR_WORKSPACE before
 *    anything is launched; use fa_bwd with your own workspace for those.
 *  - Nothing is allocated: no cudaMalloc, cudaFree or allocating library routine.
 *  - Every call looks up the scratch array's device address in the current
 *    device's context (cudaGetSymbolAddress, which allocates nothing). The first
 *    call on a device may load the library's device code there; make that first
 *    call before any stream capture.
 *  - All calls on a device share the one scratch array, which keeps whatever the
 *    last call left in it (the backward re-initialises what it needs). Two calls
 *    whose executions overlap on the GPU (different streams, no ordering between
 *    them) race on the scratch and give wrong gradients: order them on one stream
 *    or with events.
 */
#define FA_BWD_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* out,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                         int H, int N, int d, int causal, float scale, void* stream);

/* Bytes of device workspace fa_decode needs (split partials); may be 0. Depends on
 * the current device's SM count, so query it on the device that will run. */
size_t fa_decode_workspace_size(int B, int H, int Ncap, int d);

/*
 * One KV-cache decode step (flash_attn_with_kvcache, section 推理优化与KV缓存 of
 * "FlashAttention与MindSpore 2.0全场景融合方案"):
 *   q                : [B, 1, H, d] bf16 (read)
 *   k_cache, v_cache : [B, Ncap, H, d] bf16; rows >= the valid length are ignored
 *   cache_seqlens    : [B] int32 DEVICE array, valid rows before this step
 *   k_new, v_new     : [B, 1, H, d] bf16 or both NULL. When given, they are written
 *                      into the caches at row cache_seqlens[b] and the query attends
 *                      cache_seqlens[b] + 1 rows; otherwise cache_seqlens[b] rows.
 *                      cache_seqlens itself is not modified.
 *   out              : [B, 1, H, d] bf16 (written); lse : [B, H] fp32 or NULL
 *   workspace        : >= fa_decode_workspace_size(B,H,Ncap,d) bytes (may be NULL
 *                      when that size is 0), 256-byte aligned.
 * A batch entry with no valid row gets out = 0 and lse = -inf. A cache_seqlens
 * value < 0 or > Ncap, or == Ncap with k_new given, is recorded as
 * FA_ERR_DEVICE_INPUT in the device status word; that entry then attends nothing
 * and appends nothing.
 */
fa_status fa_decode(const void* q, void* k_cache, void* v_cache, const int* cache_seqlens,
                    const void* k_new, const void* v_new, void* out, float* lse, int B, int H,
                    int Ncap, int d, int causal, float scale, void* workspace,
                    size_t workspace_bytes, void* stream);

/*
 * The same decode step over a paged cache ("突破AI算力瓶颈：FlashAttention与MindSpore
 * 2.0全场景融合方案": the KV cache of section 推理优化与KV缓存 is stored in pages to avoid
 * fragmentation, and the paged cache is what its list of advantages credits for 100K+
 * sequences): the caches are a pool of fixed-size pages shared by the batch,
 *   k_pages, v_pages : [num_pages, page_size, H, d] bf16
 *   block_table      : [B, max_blocks] int32 DEVICE array; row r of sequence b is row
 *                      r % page_size of page block_table[b][r / page_size]
 * page_size is a power of two; the logical capacity is max_blocks * page_size and
 * plays the role of Ncap (a cache_seqlens value above it, or equal to it with k_new
 * given, is FA_ERR_DEVICE_INPUT). The appended row goes to its page in place. A
 * block-table entry that a row needs and that lies outside [0, num_pages) is recorded
 * as FA_ERR_DEVICE_INPUT and that row is never read or written (it counts as masked).
 * Other arguments, results and errors as fa_decode; no workspace is needed.
 */
fa_status fa_decode_paged(const void* q, void* k_pages, void* v_pages, const int* block_table,
                          int max_blocks, int page_size, int num_pages, const int* cache_seqlens,
                          const void* k_new, const void* v_new, void* out, float* lse, int B,
                          int H, int d, int causal, float scale, void* stream);

/* Message for the last non-OK status returned on the calling host thread. */
const char* fa_last_error(void);

/*
 * Folds one partial attention result into a running one, for attention split over
 * sequence shards (the ring sequence-parallel mode of "Flash-Attention 2/3在ms-swift中
 * 的集成与性能提升", section on distributed training: each device attends its query
 * shard to one key/value shard at a time and the results are combined). Both results
 * are normalised over their own keys; the merge is the stable per-block combination of
 * "FlashAttention优化Transformer显存与计算效率" section 2.2.2 in log space:
 *   LSE = log(e^lse_acc + e^lse_part),
 *   O   = e^(lse_acc - LSE) * O_acc + e^(lse_part - LSE) * O_part.
 *   o_acc    : [B, N, H, d] fp32 (read, written)   lse_acc  : [B, H, N] fp32 (read, written)
 *   o_part   : [B, N, H, d] bf16 (read)             lse_part : [B, H, N] fp32 (read)
 *   out      : [B, N, H, d] bf16 copy of the merged output (written), or NULL
 * Start from o_acc = 0 and lse_acc = -inf. A row where both LSEs are -inf keeps O_acc and
 * -inf. Errors as fa_fwd.
 */
fa_status fa_merge_partials(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                            void* out, int B, int N, int H, int d, void* stream);

/*
 * Running fp32 sum of bf16 partial results, for the backward of attention split over
 * sequence shards (the ring sequence-parallel mode of "Flash-Attention 2/3在ms-swift中
 * 的集成与性能提升", section on distributed training). With the forward's LSE and output
 * of every query row given, the recomputed backward ("ms-swift长文本训练优化，Flash-
 * Attention显存省一半" section 1.2) of one query shard against one key/value shard
 * (fa_bwd_ex) yields that pair's terms of dQ, dK and dV; each gradient is the sum of
 * its terms over the other operand's shards.
 *   acc  : n fp32 (read, written)      acc[i] += (float)part[i]  when part != NULL
 *   part : n bf16 (read), or NULL
 *   out  : n bf16 (written), or NULL   out[i] = bf16_rne(acc[i]) after the addition
 * At least one of part and out is non-NULL; n >= 0 is a multiple of 8 (n = 0 is a
 * no-op); all three pointers are 16-byte aligned device memory, any layout (the
 * operation is elementwise). Errors: FA_ERR_INVALID_ARG for a bad n, pointer or
 * alignment, before any launch; FA_ERR_UNSUPPORTED off sm_100; FA_ERR_CUDA for a
 * launch error.
 */
fa_status fa_accumulate(float* acc, const void* part, void* out, long long n, void* stream);

/*
 * Synchronises `stream`, then reads and clears the device status word of the
 * current device. Returns FA_OK, FA_ERR_TIMEOUT, FA_ERR_DEVICE_INPUT or FA_ERR_CUDA.
 * If site_out / info_out are non-NULL they receive the reporting site id and an
 * extra value (the CTA or batch index).
 */
fa_status fa_device_status(void* stream, unsigned int* site_out, unsigned int* info_out);

/*
 * Diagnostic: launches one CTA that waits on a barrier nothing will ever complete,
 * with its wait limit set to about `limit_cycles` clock cycles (clamped to
 * [1e3, 4e9]). The kernel gives up, records FA_ERR_TIMEOUT in the device status
 * word and exits; it exists so tests can check the timeout path without hanging
 * or faulting a GPU.
 */
fa_status fa_debug_timeout_probe(long long limit_cycles, void* stream);

/* Library ABI version (incremented on any signature change). */
int fa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */

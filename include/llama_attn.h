/*
 * llama_attn.h -- C ABI of libllama_attn.so: LLaMA-style self-attention on one
 * B200 GPU (sm_100a), prefill over a full sequence and single-token decode
 * against a KV cache.
 *
 * The operation (cited by page title and section):
 *   "[HuggingFace Transformers] LlamaAttention source walkthrough"
 *   (blog.csdn.net), section 1.2 steps 2-5 and section 2 forward() steps 2-6:
 *     out_h = softmax(scale * Q'_h K'_{kv(h)}^T + mask) V_{kv(h)},
 *     heads concatenated in order 0..H-1 on the last dimension,
 *   where Q' and K' are Q and K rotated by RoPE (step 3, rotate-half form
 *   x*cos + rotate_half(x)*sin, rotate_half(x) = [-x[D/2:], x[:D/2]]), and
 *   kv(h) = h / (n_heads / n_kv_heads) is the repeat_kv head map of step 4
 *   ("Llama2 Transformer architecture and optimisation practice" (lpqz.cn),
 *   section 2.1: query heads share one K/V head per group).  The softmax is
 *   computed in fp32 (step 5.2).  Decode is the "KV cache" case of
 *   "LLaMA2 large language model architecture analysis"
 *   (obsidian-quartz-blog), section "KV cache": one query row per sequence
 *   attends to every cached key; nothing is masked.
 *
 * Entry points:
 *   llama_rope_table            cos/sin tables from positions (theta, linear factor)
 *   llama_rope_table_ntk        the same with NTK-aware base scaling
 *   llama_attn_qkv_rope         q/k/v projection GEMM with RoPE in its epilogue
 *   llama_attn_out_proj         output projection GEMM
 *   llama_attn_prefill          full-sequence attention (causal or not, optional mask)
 *   llama_attn_prefill_window   causal prefill with a sliding window
 *   llama_attn_prefill_varlen   prefill of a right-padded batch (per-entry lengths)
 *   llama_attn_prefill_packed   prefill of packed sequences (cu_seqlens offsets)
 *   llama_attn_decode           one query token per sequence against a KV cache
 *   llama_attn_decode_append    the same step with the token's own K/V appended
 *   llama_attn_decode_noalloc   decode on a static scratch (no caller workspace)
 *   plus workspace sizes, the device status word, failure-detection
 *   self-tests, status strings, ABI version.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers, contiguous, row-major, owned by
 *     the caller, and must be 16-byte aligned.  The library never allocates
 *     device memory and never frees what it is given.
 *   - All work is enqueued on `cuda_stream` (a cudaStream_t; NULL = legacy
 *     default stream) and the call returns without synchronising.  Stream
 *     order is kept: the decode kernels and the RoPE table kernel launch as
 *     programmatic dependents of the preceding grid (their blocks may become
 *     resident early) but wait on the device for it to finish before they
 *     read or write any memory.  The
 *     decode combine and the RoPE table kernels allow their own programmatic
 *     dependents to launch early; a caller kernel launched with the
 *     programmatic-serialization attribute after them must wait
 *     (griddepcontrol.wait / cudaGridDependencySynchronize) before reading
 *     their outputs, as for any such launch.
 *   - cos/sin rows are LLaMA RoPE table rows: the second half of a row repeats
 *     the first (columns i and i + head_dim/2 hold the same value, because the
 *     table concatenates the frequencies with themselves), as llama_rope_table
 *     writes them.  Kernels may read either copy (the bf16 prefill kernel
 *     reads only the first half); rows whose halves differ are not supported
 *     and are not detected.
 *   - `dtype` (llama_dtype) applies to q, k, v, the caches and out together.
 *     LLAMA_DT_BF16 runs the tensor-core kernels (tcgen05 prefill, mma decode)
 *     with fp32 accumulation and an fp32 softmax; the probabilities are
 *     rounded to bf16 before the P.V product.  LLAMA_DT_F32 runs the fp32
 *     CUDA-core kernels (no TF32 anywhere).
 *   - Return value is an llama_status.  Arguments are checked on the host
 *     before anything is enqueued; on a non-zero status nothing was launched
 *     unless the status is LLAMA_ERR_CUDA (launch failure).
 *   - Device-side waits are bounded: a kernel whose pipeline wait runs out
 *     (about 2 s) records LLAMA_ERR_DEVICE_TIMEOUT in a device status word and
 *     returns; llama_attn_device_status() reads and clears it.
 */
#ifndef LLAMA_ATTN_H
#define LLAMA_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { LLAMA_DT_F32 = 0, LLAMA_DT_BF16 = 1 } llama_dtype;

typedef enum {
  LLAMA_OK = 0,
  LLAMA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, divisibility, misalignment */
  LLAMA_ERR_UNSUPPORTED = 2,   /* valid request this build has no kernel for (head_dim) */
  LLAMA_ERR_CUDA = 3,          /* a CUDA runtime/driver call or launch failed */
  LLAMA_ERR_DEVICE_TIMEOUT = 4 /* a kernel's bounded wait ran out (see above) */
} llama_status;

/*
 * RoPE cos/sin tables ("[HuggingFace Transformers] LlamaAttention source
 * walkthrough", section 2 step 3: cos, sin = rotary_emb(x, position_ids), from
 * rope_theta; linear scaling from "Llama2 Transformer architecture and
 * optimisation practice", section 6.1).
 *   pos      device int64 [bsz * seq] position ids
 *   cos, sin device fp32 [bsz * seq, head_dim] outputs.  For i < head_dim/2:
 *            angle = (pos / pos_scale_factor) * theta^(-2i/head_dim), computed
 *            in fp64 and stored as fp32 in columns i and i + head_dim/2.
 * Errors: INVALID_ARG for null pointers, bsz/seq < 1, odd or non-positive
 * head_dim, theta <= 0, pos_scale_factor <= 0.
 */
int llama_rope_table(const long long* pos, int bsz, int seq, int head_dim, double theta,
                     double pos_scale_factor, float* cos, float* sin, void* cuda_stream);

/*
 * RoPE table with NTK-aware scaling: as llama_rope_table with no position
 * scaling and the base raised to theta * alpha^(head_dim / (head_dim - 2)),
 * which keeps the highest frequency and divides the lowest by exactly alpha.
 * "Llama2 Transformer architecture and optimisation practice" section 6.1
 * names adjusting the base frequency for longer contexts without a formula;
 * this is the published NTK-aware rule.  The tables feed every attention entry
 * point unchanged.
 * Errors: as llama_rope_table, plus INVALID_ARG for alpha <= 0, head_dim < 4
 * or a base that overflows.
 */
int llama_rope_table_ntk(const long long* pos, int bsz, int seq, int head_dim, double theta,
                         double alpha, float* cos, float* sin, void* cuda_stream);

/*
 * Q/K/V projection with RoPE in the GEMM epilogue ("[HuggingFace Transformers]
 * LlamaAttention source walkthrough", section 2 forward() steps 1-3: project,
 * view per head, rotate q and k).  One tcgen05 GEMM x . w_qkv^T whose output
 * columns are the heads of q, k and v; q and k heads are rotated with the
 * token's cos/sin row before they are stored, so the results feed the
 * attention entry points with cos = sin = NULL.
 *   x        bf16 [tokens, hidden]
 *   w_qkv    bf16 [(n_heads + 2 n_kv_heads) head_dim, hidden]: the rows of
 *            W_q, then W_k, then W_v (the nn.Linear weight layout)
 *   cos, sin fp32 [tokens, head_dim] (llama_rope_table of the tokens'
 *            positions) or both NULL (no rotation)
 *   q        bf16 [tokens, n_heads, head_dim]; k, v bf16 [tokens, n_kv_heads, head_dim]
 * bf16 only.  Errors: INVALID_ARG for a NULL or misaligned pointer, tokens or
 * hidden < 1, hidden not a multiple of 8, a bad head split; UNSUPPORTED for
 * fp32 or head_dim other than 64 / 128.
 */
int llama_attn_qkv_rope(const void* x, const void* w_qkv, const float* cos, const float* sin,
                        int tokens, int hidden, int n_heads, int n_kv_heads, int head_dim,
                        void* q, void* k, void* v, int dtype, void* cuda_stream);

/*
 * Output projection y = attn . w_o^T (section 2 forward() step 7, o_proj) on
 * the same tcgen05 GEMM with a plain epilogue.
 *   attn     bf16 [tokens, in_dim] (the attention output, heads concatenated)
 *   w_o      bf16 [out_dim, in_dim]
 *   y        bf16 [tokens, out_dim]
 * bf16 only.  Errors: INVALID_ARG for a NULL or misaligned pointer, a size < 1
 * or in_dim / out_dim not a multiple of 8; UNSUPPORTED for fp32.
 */
int llama_attn_out_proj(const void* attn, const void* w_o, int tokens, int in_dim, int out_dim,
                        void* y, int dtype, void* cuda_stream);

/* Device bytes of workspace llama_attn_prefill needs for this shape (0 when
 * no RoPE or dtype is fp32).  has_rope: whether cos/sin will be passed. */
size_t llama_attn_prefill_workspace_bytes(int bsz, int n_heads, int n_kv_heads, int seq,
                                          int head_dim, int dtype, int has_rope);

/*
 * Full-sequence (prefill) attention.
 *   q        [bsz, seq, n_heads, head_dim]      (projection output viewed per
 *   k, v     [bsz, seq, n_kv_heads, head_dim]    head, no transpose: step 2)
 *   cos, sin fp32 [bsz, seq, head_dim] or both NULL for no RoPE.  Applied to q
 *            and k (never v) as x*cos + rotate_half(x)*sin, elementwise.
 *   scale    multiplies q.k (usually 1/sqrt(head_dim), step 5.1)
 *   causal   non-zero: query i sees keys j <= i (sequence index)
 *   out      [bsz, seq, n_heads * head_dim], head h at columns [h*D, (h+1)*D)
 *   add_mask fp32 [bsz, 1, seq, seq] or NULL; added to scale*q.k (step 5.1),
 *            on top of `causal` when both are given.  A row whose keys are all
 *            masked (-inf) yields zeros.
 *   workspace / workspace_bytes: caller-owned device scratch of at least
 *            llama_attn_prefill_workspace_bytes(...) bytes (may be NULL if 0).
 * Errors: INVALID_ARG for null required pointers, bsz/seq/heads < 1,
 * n_heads % n_kv_heads != 0, odd head_dim, exactly one of cos/sin NULL,
 * non-finite scale, misaligned pointers, too small a workspace, unknown
 * dtype; UNSUPPORTED for head_dim not in {64, 128}; CUDA for launch errors.
 */
int llama_attn_prefill(const void* q, const void* k, const void* v, const float* cos,
                       const float* sin, int bsz, int n_heads, int n_kv_heads, int seq,
                       int head_dim, float scale, int causal, void* out,
                       const float* add_mask, int dtype, void* workspace,
                       size_t workspace_bytes, void* cuda_stream);

/*
 * Causal prefill with a sliding window: query i attends to keys j with
 * i - window < j <= i.  The flash-attention call of "`llama.py` -- LLaMA
 * attention layer Ulysses SP adaptation" and of "[HuggingFace Transformers]
 * LlamaAttention source walkthrough" (forward(), the flash-attention branch)
 * passes the model's sliding_window without defining it; this is the reading
 * used by models that set it (a window of keys ending at the query).  K/V
 * tiles wholly before a query block's window are neither loaded nor
 * multiplied.
 *   window     >= 1 keys, the query's own included; window >= seq is plain
 *              causal attention (bit-identical to llama_attn_prefill)
 *   everything else as llama_attn_prefill with causal = 1 and no mask
 * bf16 only.  Errors: as llama_attn_prefill, plus INVALID_ARG for window < 1,
 * and UNSUPPORTED for fp32.
 */
int llama_attn_prefill_window(const void* q, const void* k, const void* v, const float* cos,
                              const float* sin, int bsz, int n_heads, int n_kv_heads, int seq,
                              int head_dim, float scale, int window, void* out, int dtype,
                              void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * Prefill of a right-padded batch: batch entry b holds seq_lens[b] valid
 * tokens at rows [0, seq_lens[b]) of the [bsz, seq, ...] tensors.  The
 * flash-attention call of "`llama.py` -- LLaMA attention layer Ulysses SP
 * adaptation" and of "[HuggingFace Transformers] LlamaAttention source
 * walkthrough" (forward(), the flash-attention branch) receives the batch's
 * attention_mask for this; here the valid lengths stand for a padding mask
 * whose ones are a prefix of each row.  Each valid query attends only its own
 * entry's valid keys (with causal, keys j <= i); output rows at or past
 * seq_lens[b] are zero.  Work on padded rows is skipped tile by tile.
 *   seq_lens   device int32 [bsz]; values are clamped to [0, seq] on the device.
 *              Padded rows of q, k and v may hold anything, NaN included.
 *   everything else as llama_attn_prefill (no additive mask)
 * bf16 only.  Errors: as llama_attn_prefill, plus INVALID_ARG for a NULL or
 * misaligned seq_lens, and UNSUPPORTED for fp32.
 */
int llama_attn_prefill_varlen(const void* q, const void* k, const void* v, const float* cos,
                              const float* sin, const int* seq_lens, int bsz, int n_heads,
                              int n_kv_heads, int seq, int head_dim, float scale, int causal,
                              void* out, int dtype, void* workspace, size_t workspace_bytes,
                              void* cuda_stream);

/*
 * Prefill of packed sequences (the layout the flash-attention call of
 * "`llama.py` -- LLaMA attention layer Ulysses SP adaptation" reaches once a
 * padded batch has been unpadded): sequence s holds tokens
 * [cu_seqlens[s], cu_seqlens[s + 1]) of the packed tensors, and each token
 * attends only to its own sequence's tokens (with causal, those at or before
 * it).  Every token row of out is written by its own sequence.
 *   q            [total_tokens, n_heads, head_dim]
 *   k, v         [total_tokens, n_kv_heads, head_dim]
 *   cos, sin     fp32 [total_tokens, head_dim] (each token's own position) or NULL
 *   cu_seqlens   device int32 [n_seqs + 1], non-decreasing from 0 to total_tokens;
 *                values are clamped to [0, total_tokens] on the device
 *   max_seqlen   >= every sequence length (longer sequences are cut to it:
 *                their later rows are not computed)
 *   out          [total_tokens, n_heads * head_dim]
 *   workspace    llama_attn_prefill_workspace_bytes(1, n_heads, n_kv_heads,
 *                total_tokens, head_dim, dtype, cos != NULL) bytes
 * bf16 only.  Errors: as llama_attn_prefill, plus INVALID_ARG for a NULL or
 * misaligned cu_seqlens, total_tokens < 1 or max_seqlen < 1, and UNSUPPORTED
 * for fp32.
 */
int llama_attn_prefill_packed(const void* q, const void* k, const void* v, const float* cos,
                              const float* sin, const int* cu_seqlens, int n_seqs,
                              int total_tokens, int max_seqlen, int n_heads, int n_kv_heads,
                              int head_dim, float scale, int causal, void* out, int dtype,
                              void* workspace, size_t workspace_bytes, void* cuda_stream);

/* Device bytes of workspace llama_attn_decode needs (split-KV partial results). */
size_t llama_attn_decode_workspace_bytes(int bsz, int n_heads, int max_cache_len, int head_dim);

/*
 * Single-token decode against a KV cache.
 *   q          [bsz, n_heads, head_dim], NOT rotated: the kernel rotates it with
 *              cos/sin (the row at the query's position)
 *   k_cache    [bsz, n_kv_heads, max_cache_len, head_dim], keys already rotated
 *   v_cache    [bsz, n_kv_heads, max_cache_len, head_dim]
 *   cache_lens device int32 [bsz]: rows [0, cache_lens[b]) are attended.  Values
 *              are clamped to [0, max_cache_len] on the device; a length of 0
 *              yields a zero output row.  Rows at or past the length are never
 *              read into the result (they may hold anything, NaN included).
 *   cos, sin   fp32 [bsz, head_dim] or both NULL (no RoPE on q)
 *   out        [bsz, n_heads * head_dim]
 *   workspace  caller-owned device scratch of at least
 *              llama_attn_decode_workspace_bytes(...) bytes
 * Errors: as llama_attn_prefill, plus INVALID_ARG for max_cache_len < 1 or a
 * NULL cache_lens, and UNSUPPORTED for bf16 with bsz > 4096 (the bf16 kernel
 * keeps a per-batch prefix of chunk counts in shared memory).
 */
int llama_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                      const int* cache_lens, const float* cos, const float* sin, int bsz,
                      int n_heads, int n_kv_heads, int max_cache_len, int head_dim,
                      float scale, void* out, void* workspace, size_t workspace_bytes,
                      int dtype, void* cuda_stream);

/*
 * One decode step with the new token's own key and value ("LLaMA2 large
 * language model architecture analysis", section "KV cache": the step's key
 * and value are appended to the cache, then the query attends over every row
 * including its own).  For each batch entry b, with p = min(max(cache_lens[b],
 * 0), max_cache_len - 1) the new token's row:
 *   k_cache[b, g, p, :] = RoPE(k_new[b, g, :]) rotated with cos/sin[b] (the
 *                         query's position, which is the new token's), rounded
 *                         to bf16; v_cache[b, g, p, :] = v_new[b, g, :]
 *   out[b, h*D:(h+1)*D] = attention of RoPE(q[b, h]) over cache rows 0..p of
 *                         K/V head h / (n_heads / n_kv_heads)
 * in one pass (no separate append launch).
 *   q            [bsz, n_heads, head_dim], not rotated
 *   k_new, v_new [bsz, n_kv_heads, head_dim]; k_new not rotated
 *   k_cache, v_cache  as llama_attn_decode, written at row p (and nowhere else)
 *   cache_lens   device int32 [bsz], read only: the caller advances it
 *   cos, sin, out, workspace  as llama_attn_decode
 * bf16 only.  Errors: as llama_attn_decode, plus INVALID_ARG for a NULL or
 * misaligned k_new / v_new, and UNSUPPORTED for fp32.  A batch entry whose
 * cache is full (cache_lens[b] >= max_cache_len) has its last row replaced.
 */
int llama_attn_decode_append(const void* q, const void* k_new, const void* v_new,
                             void* k_cache, void* v_cache, const int* cache_lens,
                             const float* cos, const float* sin, int bsz, int n_heads,
                             int n_kv_heads, int max_cache_len, int head_dim, float scale,
                             void* out, void* workspace, size_t workspace_bytes, int dtype,
                             void* cuda_stream);

/*
 * Single-token decode for callers that cannot allocate device memory.  The
 * pages have no counterpart to this entry point; it exists for integrations
 * that hand the library only their input and output buffers -- hosts that
 * reserve all device memory up front and forbid further cudaMalloc (which
 * could also synchronise the device mid-step), or plugin interfaces that
 * provide no workspace.  It computes exactly what llama_attn_decode computes,
 * with the same arguments minus the workspace.
 *
 * Scratch: a file-scope device array of 16 MiB inside the library, which every
 * GPU that loads the library holds until the process exits.  A request needing
 * more than that (see llama_attn_decode_workspace_bytes) is rejected with
 * LLAMA_ERR_INVALID_ARG before anything is enqueued; use llama_attn_decode
 * with a caller workspace instead.  fp32 requests need no scratch.
 * Every call looks up the array's device address on the current device (one
 * cudaGetSymbolAddress, which allocates nothing).  The first call on a device
 * may load the library's device code there: make it before any stream
 * capture on that device.
 * Every call on a device shares the one array and leaves its last contents
 * behind (each call writes every scratch entry it later reads, so nothing has
 * to start at zero).  Calls whose kernels overlap on the GPU -- concurrent
 * streams, or several host threads -- race on the array: serialise them.
 */
int llama_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                              const int* cache_lens, const float* cos, const float* sin, int bsz,
                              int n_heads, int n_kv_heads, int max_cache_len, int head_dim,
                              float scale, void* out, int dtype, void* cuda_stream);

/* Synchronises `cuda_stream`, then reads and clears the device status word of
 * the current device.  Returns LLAMA_OK, LLAMA_ERR_DEVICE_TIMEOUT, or
 * LLAMA_ERR_CUDA if the synchronisation itself failed. */
int llama_attn_device_status(void* cuda_stream);

/*
 * Self-tests of failure detection.  The pages have no counterpart; these two
 * calls let a test (or a deployment's health check) see both failure paths
 * of the library work without faulting the GPU.
 *
 * llama_attn_selftest_wait_timeout: launches one warp that waits on a shared-
 * memory barrier nothing ever arrives on, with the given limit in
 * microseconds (1 .. 1000000) instead of the pipelines' 2 s.  The wait runs
 * out, records LLAMA_ERR_DEVICE_TIMEOUT in the device status word and the
 * kernel returns, with no copy or MMA in flight.  Returns LLAMA_OK once the
 * launch is enqueued (INVALID_ARG for a limit outside the range); a following
 * llama_attn_device_status() reports LLAMA_ERR_DEVICE_TIMEOUT, the next one
 * LLAMA_OK.
 *
 * llama_attn_selftest_launch_error: asks for a kernel launch with an invalid
 * block size, which the CUDA runtime refuses on the host; returns
 * LLAMA_ERR_CUDA, as any library call whose launch fails does.  Nothing
 * reaches the GPU and the context stays usable.
 */
int llama_attn_selftest_wait_timeout(unsigned int limit_us, void* cuda_stream);
int llama_attn_selftest_launch_error(void* cuda_stream);

/* Static, NUL-terminated description of a status code. */
const char* llama_attn_status_string(int status);

/* ABI version (major * 100 + minor): 120 = 1.2, the entry points above. */
int llama_attn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LLAMA_ATTN_H */

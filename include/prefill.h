/*
 * prefill.h -- C ABI of libprefill: causal prefill attention (MHA / GQA) for
 * NVIDIA B200 (sm_100a), fused with the paged KV-cache write.
 *
 * What a call computes, for every sequence i of a packed batch, every query
 * row a of that sequence and every query head h:
 *
 *   P    = ctx_i + a                  absolute position (ctx_i = 0 for prefill_attn)
 *   g    = h / (n_head / n_kv_head)   kv head shared by a contiguous group of query heads
 *   s_j  = scale * <q[a][h], k_j[g]>  for keys j = 0 .. P   (causal: later keys are skipped)
 *   out[a][h] = sum_j softmax(s)_j * v_j[g]
 *
 * and it writes every token's K and V rows into its page of the KV cache.
 *
 * Sources (page address and section):
 *   hncyxsy.com/news/270449 §2.2  head split: (s, h) viewed as (s, n_head, head_dim), head_dim last
 *   hncyxsy.com/news/270449 §2.3  per-head scores, causal upper-triangle mask, softmax, times V
 *   hncyxsy.com/news/270449 §3.1  scores divided by sqrt(head_dim); mask by block-index control flow
 *   hncyxsy.com/news/270449 §3.2  online softmax: per-block max and exp-sum, old results rescaled
 *   hncyxsy.com/news/270449 §3.3  heads merged back to (s, h) by flattening (s, n_head, head_dim)
 *   hncyxsy.com/news/270449 §3.4  GQA: several query heads share one K/V head
 *   hncyxsy.com/news/270449 §4.2  KV cache in fixed-size blocks; the write is fused, not a copy kernel
 *   hncyxsy.com/news/270449 §4.3  query blocks x kv blocks; skip / unmasked / column-masked blocks
 *   hncyxsy.com/news/227904 §2.1  chunked prefill: a chunk attends to all earlier K/V
 *   hncyxsy.com/news/227904 §3.4  page table maps a sequence's logical pages to physical blocks
 *   lnwmold.com/news/496245 §3.3  block size 16, prefill chunk 512 (workload shapes)
 *
 * Layouts (all row-major, contiguous, little-endian bf16 = IEEE bfloat16 bits):
 *   q, out    [total_tokens][n_head][head_dim]
 *   k, v      [total_tokens][n_kv_head][head_dim]
 *   kv_cache  [num_blocks][2][block_size][n_kv_head][head_dim]   ([.][0] = K page, [.][1] = V page)
 *   block_table  int32 [num_seqs][max_blocks_per_seq]; logical page p of sequence i
 *                (positions p*block_size .. p*block_size+block_size-1) lives in
 *                physical block block_table[i][p].  Entries past a sequence's last
 *                page are never read.
 *   cu_seqlens   int32 [num_seqs + 1]; sequence i owns packed rows
 *                cu_seqlens[i] .. cu_seqlens[i+1]-1 (non-decreasing, cu_seqlens[0] = 0).
 *
 * Ownership: every pointer argument is caller-owned DEVICE memory, except where
 * stated.  Calls enqueue their work asynchronously on `stream` (the legacy
 * default stream if NULL).  They write `out`, the cache slots of the tokens they
 * process, and `*status_dev`; nothing else of the caller's.  Inputs must stay
 * valid until the work on `stream` completes.
 *
 * Split-KV workspace: when a call has fewer work items than the GPU has SMs
 * (typically a chunked-prefill chunk attending to a long cached prefix), the
 * kv range of each item is split across CTAs and the partial results are
 * merged by a second kernel on the same stream.  The partials live in a device
 * workspace that the library owns: allocated on the first such call for a
 * given (device, stream) and kept for later calls, grown when a larger call
 * needs more.  Allocation and growth are stream-ordered (cudaMallocAsync, and
 * cudaFreeAsync of the smaller buffer, on `stream`), so a call never blocks the
 * host or waits for the stream; calls that do not split allocate nothing.
 * Size: splits x total rows x n_head x (head_dim + 2) x 4 bytes + 4 bytes per
 * row, splits <= 8.
 * If the allocation fails the call runs unsplit.  prefill_attn_chunked_noalloc
 * is the chunked call that allocates nothing.
 *
 * Errors: argument problems that the host can see are returned synchronously
 * and nothing is launched.  Problems only the device can see (a block-table
 * entry outside [0, num_blocks), a sequence longer than the bound given, a
 * decreasing cu_seqlens, a pipeline wait that ran past its limit) make the
 * affected work skip its memory accesses and set `*status_dev` to the first
 * such code (atomic compare-and-swap from PREFILL_OK); the caller zeroes it
 * before the call and reads it after synchronising.  With status_dev == NULL
 * such problems are still skipped but not reported.
 *
 * Preconditions (stated, not checked): no physical block appears twice in the
 * block table (within or across sequences); input values are finite.
 */
#ifndef LIBPREFILL_PREFILL_H
#define LIBPREFILL_PREFILL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Raw bfloat16 storage (the 16 high bits of an IEEE binary32). */
typedef uint16_t prefill_bf16;
/* Same object as a CUDA runtime cudaStream_t / driver CUstream. */
typedef struct CUstream_st *prefill_stream_t;

typedef enum {
    PREFILL_OK = 0,
    PREFILL_ERR_NULL = 1,         /* a required pointer is NULL */
    PREFILL_ERR_SHAPE = 2,        /* inconsistent sizes or a sequence longer than the bound given */
    PREFILL_ERR_UNSUPPORTED = 3,  /* head_dim, block_size or scale outside the supported set */
    PREFILL_ERR_BLOCK_TABLE = 4,  /* block-table entry outside [0, num_blocks) or table too short */
    PREFILL_ERR_CUDA = 5,         /* launch or driver failure */
    PREFILL_ERR_TIMEOUT = 6,      /* a device-side pipeline wait ran past its limit (about one second) */
    PREFILL_ERR_ALIGNMENT = 7,    /* a pointer is not 16-byte aligned */
    PREFILL_ERR_SCRATCH_LIMIT = 8 /* reserved: no current entry point returns it (the value stays assigned) */
} prefill_status;

/*
 * prefill_attn -- causal prefill attention over whole prompts, fused with the
 * paged KV write (hncyxsy.com/news/270449 §3.1-§4.3; hncyxsy.com/news/227904 §3.4).
 *
 *   q, k, v        device, layouts above, total_tokens rows each
 *   total_tokens   rows in q/k/v/out (= cu_seqlens[num_seqs]); 0 is a no-op
 *   cu_seqlens     device int32 [num_seqs + 1]
 *   num_seqs       >= 1 (0 is a no-op)
 *   max_seqlen     upper bound on every sequence length (host value; sizes the grid)
 *   n_head, n_kv_head   n_head % n_kv_head == 0
 *   head_dim       64 or 128
 *   scale          finite, > 0 (normally 1/sqrt(head_dim))
 *   out            device, written: [total_tokens][n_head][head_dim] bf16
 *   kv_cache       device, written at the slots of this call's tokens only
 *   num_blocks     physical blocks in kv_cache (>= 1)
 *   block_table    device int32 [num_seqs][max_blocks_per_seq]
 *   block_size     16, 32, 64 or 128 tokens per block
 *   status_dev     device int32 (nullable), see Errors above
 *   stream         CUDA stream to enqueue on
 * Requires max_seqlen <= max_blocks_per_seq * block_size.
 * Returns a prefill_status.
 */
int prefill_attn(const prefill_bf16 *q, const prefill_bf16 *k, const prefill_bf16 *v,
                 int total_tokens, const int32_t *cu_seqlens, int num_seqs, int max_seqlen,
                 int n_head, int n_kv_head, int head_dim, float scale,
                 prefill_bf16 *out,
                 prefill_bf16 *kv_cache, int num_blocks,
                 const int32_t *block_table, int max_blocks_per_seq, int block_size,
                 int32_t *status_dev, prefill_stream_t stream);

/*
 * prefill_attn_chunked -- chunked prefill (hncyxsy.com/news/227904 §2.1): each
 * sequence's query chunk attends to the context_lens[i] tokens already in the
 * cache (gathered through block_table) plus itself, causally, with the chunk
 * aligned at the end: chunk row a sits at absolute position context_lens[i] + a.
 * The chunk's own K/V are then appended to the cache at those positions.
 *
 *   q, k, v        device, the chunk's rows only: total_q rows
 *   cu_seqlens_q   device int32 [num_seqs + 1] over the chunk rows
 *   context_lens   device int32 [num_seqs]: cached tokens before each chunk
 *   max_q_len      upper bound on every chunk length (host)
 *   max_context_len  upper bound on every context length (host)
 *   the rest as for prefill_attn.
 * The cached prefix is read as it stands before the call (the slots this call
 * writes are all at positions >= context_lens[i]).
 * Requires max_q_len <= max_blocks_per_seq * block_size and max_context_len <=
 * max_blocks_per_seq * block_size; a sequence whose context_lens[i] + chunk
 * length exceeds the table is skipped on the device and reported as
 * PREFILL_ERR_BLOCK_TABLE.
 */
int prefill_attn_chunked(const prefill_bf16 *q, const prefill_bf16 *k, const prefill_bf16 *v,
                         int total_q, const int32_t *cu_seqlens_q, const int32_t *context_lens,
                         int num_seqs, int max_q_len, int max_context_len,
                         int n_head, int n_kv_head, int head_dim, float scale,
                         prefill_bf16 *out,
                         prefill_bf16 *kv_cache, int num_blocks,
                         const int32_t *block_table, int max_blocks_per_seq, int block_size,
                         int32_t *status_dev, prefill_stream_t stream);

/*
 * prefill_attn_sliding_window -- causal prefill with a sliding window
 * (lnwmold.com/news/496245 §4.1: each token attends only to its nearest W
 * predecessors, so n rows cost n*W instead of n^2 key visits).  Row a of
 * sequence i, at absolute position P = context_lens[i] + a, sees keys
 * max(0, P - window + 1) .. P: the window counts the token itself, and
 * window >= P + 1 for every row gives plain causal attention.  The KV write is
 * the same as for prefill_attn: every token of the call lands in its slot,
 * whether or not later rows still see it.
 *
 *   context_lens   device int32 [num_seqs] (chunked prefill: the window
 *                  reaches back into the cached prefix, and prefix blocks
 *                  wholly before it are not read), or NULL for plain prefill
 *                  (then max_context_len must be 0)
 *   window         keys per row, >= 1
 *   the rest as for prefill_attn_chunked.
 * Errors as for prefill_attn_chunked, plus PREFILL_ERR_SHAPE for window < 1 or
 * a non-zero max_context_len without context_lens.
 */
int prefill_attn_sliding_window(const prefill_bf16 *q, const prefill_bf16 *k, const prefill_bf16 *v,
                                int total_q, const int32_t *cu_seqlens_q, const int32_t *context_lens,
                                int num_seqs, int max_q_len, int max_context_len,
                                int n_head, int n_kv_head, int head_dim, float scale, int window,
                                prefill_bf16 *out,
                                prefill_bf16 *kv_cache, int num_blocks,
                                const int32_t *block_table, int max_blocks_per_seq, int block_size,
                                int32_t *status_dev, prefill_stream_t stream);

/*
 * paged_decode_attn -- decode attention over the paged cache (the next step
 * after prefill: hncyxsy.com/news/270449 §1.1, decode feeds only the token
 * generated last; hncyxsy.com/news/227904 §1, the step is then bound by
 * memory bandwidth, reading the KV cache).  For each sequence i, the one new
 * token at absolute position context_lens[i] attends to the context_lens[i]
 * cached tokens (gathered through block_table) and to itself; its K/V are then
 * written to their slot.  The result equals prefill_attn_chunked with one-row
 * chunks.
 *
 *   q              device bf16 [num_seqs][n_head][head_dim]: the new tokens' queries
 *   k, v           device bf16 [num_seqs][n_kv_head][head_dim]: their keys and values
 *   context_lens   device int32 [num_seqs]: cached tokens before each new one
 *   max_context_len  upper bound on every context length (host; sizes the grid)
 *   out            device, written: [num_seqs][n_head][head_dim] bf16
 *   kv_cache, num_blocks, block_table, max_blocks_per_seq, block_size,
 *   status_dev, stream   as for prefill_attn_chunked.
 * n_head / n_kv_head must be at most 16 and num_seqs at most 2048
 * (PREFILL_ERR_UNSUPPORTED otherwise).
 * Requires max_context_len + 1 <= max_blocks_per_seq * block_size.  A sequence
 * whose context length is negative or above max_context_len is skipped and
 * reported as PREFILL_ERR_SHAPE.  Contexts are split into units of >= 128
 * keys whose partial results a second kernel merges; their partials use the
 * same per-(device, stream) workspace as the prefill split-KV partials
 * (max units x num_seqs x n_head x (head_dim + 2) x 4 bytes).
 */
int paged_decode_attn(const prefill_bf16 *q, const prefill_bf16 *k, const prefill_bf16 *v,
                      const int32_t *context_lens, int num_seqs, int max_context_len,
                      int n_head, int n_kv_head, int head_dim, float scale,
                      prefill_bf16 *out,
                      prefill_bf16 *kv_cache, int num_blocks,
                      const int32_t *block_table, int max_blocks_per_seq, int block_size,
                      int32_t *status_dev, prefill_stream_t stream);

/*
 * FP8 KV cache (hncyxsy.com/news/227904 §2.3: the KV cache may stay in FP8
 * while the softmax keeps higher precision; §3.3: 1 byte per element).
 * Format e4m3 (bias 7, 3 mantissa bits, no infinities, largest finite 448).
 * The cache has the bf16 cache's layout with one byte per element,
 * uint8 [num_blocks][2][block_size][n_kv_head][head_dim], and each kv head g
 * has a K scale and a V scale (device fp32 [n_kv_head], caller-chosen, > 0):
 * an element x is stored as the code of x / scale (fp32 division, rounded to
 * the nearest code, ties to even, magnitudes beyond 448 saturated) and read as
 * code_value * scale.
 *
 * kv_cache_store_fp8 -- write a call's K/V rows (k, v [total_tokens][n_kv_head]
 * [head_dim] bf16, sequences by cu_seqlens, row a of sequence i at position
 * context_lens[i] + a, context_lens NULL meaning 0) into their FP8 cache slots.
 * Nothing else in the pool changes.  Argument checks and status codes as for
 * prefill_attn_chunked.
 */
int kv_cache_store_fp8(const prefill_bf16 *k, const prefill_bf16 *v, int total_tokens,
                       const int32_t *cu_seqlens, const int32_t *context_lens, int num_seqs,
                       int n_kv_head, int head_dim, const float *k_scale, const float *v_scale,
                       uint8_t *kv_cache_fp8, int num_blocks,
                       const int32_t *block_table, int max_blocks_per_seq, int block_size,
                       int32_t *status_dev, prefill_stream_t stream);

/*
 * paged_decode_attn_fp8 -- paged_decode_attn over an FP8 cache: the new token
 * of sequence i attends to the dequantized codes of positions
 * 0 .. context_lens[i] - 1 and to its own K/V quantized the same way (every key
 * and value the attention sees is a dequantized cache value); its codes are
 * written to its slot.  Softmax and accumulation in fp32; the products run on
 * f16 tensor-core operands (every e4m3 value is exact in f16; q is rounded to
 * f16, exact for bf16 values of magnitude 2^-14 .. 65504).  Arguments as for
 * paged_decode_attn, plus k_scale / v_scale (device fp32 [n_kv_head]).
 */
int paged_decode_attn_fp8(const prefill_bf16 *q, const prefill_bf16 *k, const prefill_bf16 *v,
                          const int32_t *context_lens, int num_seqs, int max_context_len,
                          int n_head, int n_kv_head, int head_dim, float scale,
                          const float *k_scale, const float *v_scale,
                          prefill_bf16 *out,
                          uint8_t *kv_cache_fp8, int num_blocks,
                          const int32_t *block_table, int max_blocks_per_seq, int block_size,
                          int32_t *status_dev, prefill_stream_t stream);

/*
 * prefill_attn_fp8_cache -- prefill_attn writing an FP8 cache: the same
 * attention over the bf16 inputs (out is what prefill_attn returns), with each
 * token's K/V rows stored in kv_cache_fp8 as the codes kv_cache_store_fp8
 * writes (the FP8 format above).  Two launches on `stream`: the attention
 * kernel without its cache writer, then the FP8 store kernel.  (The pages put
 * the cache write inside the attention kernel, hncyxsy.com/news/270449 §4.2;
 * for the bf16 cache that is what prefill_attn does, but quantizing inside the
 * softmax-bound kernel measured slower than the separate pass.)
 * Arguments, limits and errors as for prefill_attn, with k_scale / v_scale
 * (device fp32 [n_kv_head], > 0) and the uint8 pool in place of the bf16 one.
 * PREFILL_ERR_UNSUPPORTED when the call is beyond the work schedule that the
 * pipelined kernel keeps in shared memory (more than 4096 sequences, or a
 * max_seqlen above 524,288), where prefill_attn would run its simple kernel.
 */
int prefill_attn_fp8_cache(const prefill_bf16 *q, const prefill_bf16 *k, const prefill_bf16 *v,
                           int total_tokens, const int32_t *cu_seqlens, int num_seqs, int max_seqlen,
                           int n_head, int n_kv_head, int head_dim, float scale,
                           const float *k_scale, const float *v_scale,
                           prefill_bf16 *out, uint8_t *kv_cache_fp8, int num_blocks,
                           const int32_t *block_table, int max_blocks_per_seq, int block_size,
                           int32_t *status_dev, prefill_stream_t stream);

/*
 * prefill_attn_chunked_fp8 -- prefill_attn_chunked over an FP8 cache
 * (hncyxsy.com/news/227904 §2.1 chunked prefill; §2.3 the KV cache in FP8
 * with the softmax at higher precision).  Chunk row a of sequence i sits at
 * position context_lens[i] + a and attends to keys 0 .. context_lens[i] + a,
 * every one of them a dequantized cache value: the cached prefix's codes, and
 * the chunk's own K/V rows quantized with the same scales, as they are stored.
 * The chunk's codes are appended to kv_cache_fp8 (as kv_cache_store_fp8 writes
 * them).  Arguments, limits and errors as for prefill_attn_chunked, with
 * k_scale / v_scale (device fp32 [n_kv_head], > 0) and the uint8 pool.
 *
 * Two launches on `stream` (three when the kv ranges are split): the FP8
 * store of the chunk's codes, into the pool and into a dense per-call copy of
 * the chunk's rows; then the attention kernel, which TMA-loads every key and
 * value as e4m3 bytes -- the prefix page by page through block_table, the
 * chunk's own rows from the dense copy -- widens them to f16 in shared memory
 * (exact: an e4m3 value has at most 4 significant bits), converts q to f16 the
 * same way and runs its products on f16 tensor-core operands, with each kv
 * head's K scale folded into its scores and V scale into its output (fp32).
 * q is taken as f16: exact for bf16 values of magnitude 2^-14 .. 65504 (larger
 * magnitudes overflow; smaller ones lose low bits).  The dense copy, 2 x
 * total_q x n_kv_head x head_dim bytes, is a workspace allocated like the
 * split-KV one (first call per device and stream, grown stream-ordered, kept);
 * PREFILL_ERR_CUDA if that allocation fails.  PREFILL_ERR_UNSUPPORTED where the
 * pipelined kernel's schedule does not fit (as for prefill_attn_fp8_cache).
 */
int prefill_attn_chunked_fp8(const prefill_bf16 *q, const prefill_bf16 *k, const prefill_bf16 *v,
                             int total_q, const int32_t *cu_seqlens_q, const int32_t *context_lens,
                             int num_seqs, int max_q_len, int max_context_len,
                             int n_head, int n_kv_head, int head_dim, float scale,
                             const float *k_scale, const float *v_scale,
                             prefill_bf16 *out, uint8_t *kv_cache_fp8, int num_blocks,
                             const int32_t *block_table, int max_blocks_per_seq, int block_size,
                             int32_t *status_dev, prefill_stream_t stream);

/*
 * qkv_projection -- the fused QKV projection that feeds prefill_attn
 * (hncyxsy.com/news/270449 §4.1: the W_q, W_k, W_v blocks concatenated into
 * one GEMM that reads the activations once, its output cut by columns into
 * Q, K and V; §2.2: each reshaped to (tokens, heads, head_dim)).
 *
 *   x        device bf16 [tokens][hidden], row-major
 *   w        device bf16 [(n_head + 2 n_kv_head) head_dim][hidden]: one row per
 *            output feature (the layout of a linear layer's weight), the
 *            n_head head_dim rows of W_q first, then W_k's, then W_v's
 *   q        device, written: bf16 [tokens][n_head][head_dim]
 *   k, v     device, written: bf16 [tokens][n_kv_head][head_dim]
 * y = x w^T with fp32 accumulation, each output rounded once to bf16 (round to
 * nearest even).  Requires hidden a multiple of 64, head_dim a multiple of 32
 * and (n_head + 2 n_kv_head) head_dim a multiple of 256
 * (PREFILL_ERR_UNSUPPORTED otherwise); pointers 16-byte aligned.  Runs on the
 * tensor cores (tcgen05) with 128 x 256 output tiles (128 x 192 when that width
 * divides the output and fills the GPU's waves better); a device wait that runs
 * past its limit is reported as PREFILL_ERR_TIMEOUT in *status_dev.
 */
int qkv_projection(const prefill_bf16 *x, const prefill_bf16 *w, int tokens, int hidden,
                   int n_head, int n_kv_head, int head_dim,
                   prefill_bf16 *q, prefill_bf16 *k, prefill_bf16 *v,
                   int32_t *status_dev, prefill_stream_t stream);

/*
 * attn_out_projection -- the output projection W_o that follows prefill_attn
 * (hncyxsy.com/news/270449 §3.3: the heads' outputs merged back to (s, h) by
 * flattening (s, n_head, head_dim), head after head, so that W_o is a plain
 * GEMM whose input features run in head order; §2.3: it maps the merged
 * heads to the hidden size).
 *
 *   o        device bf16 [tokens][n_head][head_dim] (prefill_attn's out), read as
 *            [tokens][n_head * head_dim]
 *   w_o      device bf16 [hidden][n_head * head_dim]: one row per output feature
 *   y        device, written: bf16 [tokens][hidden]
 * y = o w_o^T with fp32 accumulation, each output rounded once to bf16 (round to
 * nearest even).  Requires n_head * head_dim a multiple of 64 and hidden a
 * multiple of 256 (PREFILL_ERR_UNSUPPORTED otherwise); pointers 16-byte
 * aligned.  Same tensor-core kernel, limits and error reports as qkv_projection.
 */
int attn_out_projection(const prefill_bf16 *o, const prefill_bf16 *w_o, int tokens, int n_head,
                        int head_dim, int hidden, prefill_bf16 *y,
                        int32_t *status_dev, prefill_stream_t stream);

/*
 * prefill_attn_chunked_noalloc -- prefill_attn_chunked for callers that cannot
 * let the library allocate device memory.  The pages have no counterpart: this
 * is a deployment variant of the chunked call, not a step of the method.
 *
 * prefill_attn_chunked may split long kv ranges (split-KV) and then obtains a
 * workspace with cudaMalloc.  Some callers cannot allow that: serving engines
 * that own all device memory through their own pool (an allocation behind the
 * pool's back can fail or fragment the memory it has reserved), and processes
 * whose device-memory budget is fixed at start-up.  This entry point computes
 * the same result with the same kernels, keeping the split partials in a
 * fixed device array that is part of the library: 32 MiB
 * (prefill_noalloc_scratch_bytes()) on every GPU that loads the library, held
 * until the process exits.  It calls no cudaMalloc, cudaFree or allocating
 * library routine.
 *
 *   Arguments, layouts and errors as for prefill_attn_chunked.  A call whose
 *   chosen split count would need more than the array holds -- splits x
 *   total_q x n_head x (head_dim + 2) x 4 + 4 x total_q bytes -- runs with the largest split
 *   count that fits (down to 1, which needs no scratch), so every call that
 *   prefill_attn_chunked accepts runs here too, with the same result up to
 *   the rounding order of the split merge.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) and caches it; make that first call before any stream
 * capture.  Every call uses the same array, which keeps the last call's
 * contents (nothing in it needs to start at zero: each call writes every
 * partial it later reads).  Calls whose GPU work overlaps -- on different
 * streams, or unordered from different threads -- race on the array: the
 * caller must serialise them.
 */
int prefill_attn_chunked_noalloc(const prefill_bf16 *q, const prefill_bf16 *k, const prefill_bf16 *v,
                                 int total_q, const int32_t *cu_seqlens_q, const int32_t *context_lens,
                                 int num_seqs, int max_q_len, int max_context_len,
                                 int n_head, int n_kv_head, int head_dim, float scale,
                                 prefill_bf16 *out,
                                 prefill_bf16 *kv_cache, int num_blocks,
                                 const int32_t *block_table, int max_blocks_per_seq, int block_size,
                                 int32_t *status_dev, prefill_stream_t stream);

/* Size in bytes of prefill_attn_chunked_noalloc's fixed split-KV array. */
size_t prefill_noalloc_scratch_bytes(void);

/*
 * Test hook for the failure path (no counterpart on the pages).  With enable
 * != 0, the next prefill_attn / prefill_attn_chunked launch that uses the
 * pipelined kernel withholds its first Q tile in CTA 0, so that the consumer's
 * bounded wait (about one second) expires: every role of the kernel then stops,
 * drains its copies, frees its tensor memory and returns, and *status_dev
 * reads PREFILL_ERR_TIMEOUT.  The hook resets itself after one launch.  It makes
 * no fault and no hang; it exists so tests can check that a stalled pipeline is
 * reported and that the CUDA context stays usable.
 */
void prefill_test_inject_stall(int enable);

/*
 * Test hook for the FMA-pipe exponential (no counterpart on the pages).  The
 * pipelined kernel takes one exponential in eight of an unmasked block's
 * softmax as a polynomial on the FMA pipe instead of the MUFU ex2 unit, to
 * shorten the softmax; this call applies that same device function to n floats
 * so that tests can bound its error against exp2: y[i] ~= 2^x[i] for x[i] in
 * [-125, 127] (inputs below -125 give about 2^-125).  x, y: device float [n].
 * Returns PREFILL_ERR_NULL / PREFILL_ERR_SHAPE for bad arguments, else
 * launches one small kernel on `stream`.
 */
int prefill_test_exp2_fma2(const float *x, float *y, int n, prefill_stream_t stream);

/* Human-readable name of a prefill_status value (static storage). */
const char *prefill_status_string(int status);

/*
 * Causal block rule (hncyxsy.com/news/270449 §4.3), exported so that host code
 * and tests can check the exact rule the kernels use.  Host-only, no GPU needed.
 *
 * A query block covers chunk rows [qb*bm, qb*bm + bm).  Its kv blocks are
 * numbered j = 0 .. prefill_num_kv_blocks()-1: first the cached prefix
 * (positions [j*bn, j*bn + bn) intersected with [0, ctx)), then the chunk's own
 * keys in blocks of bn aligned to the chunk start, up to the diagonal block.
 * Blocks above the diagonal are not numbered (never issued).
 *
 * prefill_kv_block_rule returns 0 if every (row < n, key) pair of block j is
 * visible (no mask), 1 if it is partly masked, -1 if j is out of range; for a
 * masked block it writes, for each row r of the query block, the number of
 * leading visible key columns to col_limit[r] (bm entries; may be NULL).
 * Its key range starts at absolute position *key_begin (may be NULL).
 *
 * Under a sliding window of `window` keys (window 0: none) the visit starts
 * at prefill_first_kv_block() instead of 0 (blocks wholly before the first
 * row's window are not issued), and prefill_kv_block_rule_window also writes
 * each row's first visible column to col_lo[r]: row r sees the columns
 * [col_lo[r], col_limit[r]) of block j.  Both return values as above.
 */
int prefill_num_kv_blocks(int qb, int ctx, int n, int bm, int bn);
int prefill_kv_block_rule(int qb, int j, int ctx, int n, int bm, int bn,
                          int32_t *col_limit, int32_t *key_begin);
int prefill_first_kv_block(int qb, int ctx, int n, int bm, int bn, int window);
int prefill_kv_block_rule_window(int qb, int j, int ctx, int n, int bm, int bn, int window,
                                 int32_t *col_lo, int32_t *col_limit, int32_t *key_begin);

#ifdef __cplusplus
}
#endif
#endif /* LIBPREFILL_PREFILL_H */

/*
 * attn_b200.h -- C ABI of libattn_b200.so: exact scaled-dot-product attention
 * on NVIDIA B200 (sm_100a).
 *
 *     O = softmax(Q K^T * scale + mask) V
 *
 * The operation is the one every source page turns on: "Attention mechanism
 * explained: from Self-Attention to Multi-Query Attention" (guijiagi.com),
 * section 2.1 (the formula) and 2.2 (masked_fill with -inf before softmax);
 * "Taking LLMs apart (2): attention by hand" (blog.kerro.cn), sections
 * "full implementation" (mask True = visible, masked logits -inf) and
 * "FlashAttention" (tiled evaluation with an online softmax gives the exact
 * same result).  Two forms are provided:
 *
 *   attn_prefill / attn_prefill_f32   tiled, FlashAttention-style prefill
 *                                     ("Attention From Scratch" project
 *                                     README, section "Flash Attention";
 *                                     the Attention-mechanism explainer,
 *                                     section 7) with causal and
 *                                     sliding-window masks ("LLM core
 *                                     technology", section "Sliding Window
 *                                     Attention") and MHA/GQA/MQA head sharing
 *                                     (explainer, sections 4-5).
 *   attn_decode_paged                 one query token per sequence against a
 *                                     paged KV cache ("Attention From
 *                                     Scratch" README, sections "KV Cache"
 *                                     and "Paged KV Cache"; "LLM core
 *                                     technology", section "PagedAttention").
 *
 * Around them:
 *
 *   attn_prefill_lse, attn_prefill_f32_lse   the same prefill, with each row's
 *                                     log-sum-exp (the README's FlashAttention
 *                                     returns the pair (output, lse)).
 *   attn_prefill_paged                chunked prefill whose keys and values sit
 *                                     in the paged cache.
 *   attn_prefill_host                 the prefill from and to host memory, its
 *                                     copies overlapped with the kernels.
 *   attn_decode_step_host             one decode step from and to host memory:
 *                                     copy in, append, decode, copy out.
 *   attn_decode_paged_fp8             the decode over a cache of 8-bit E4M3
 *                                     codes (not on the pages: a storage
 *                                     variant).
 *   attn_decode_paged_noalloc         the decode with a fixed scratch array
 *                                     instead of a workspace.
 *   attn_kv_append, attn_kv_append_fp8  write new tokens' K/V into the cache.
 *   attn_page_pool_*                  a host-side page allocator and the page
 *                                     tables it uploads.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers named q, k, v, out, k_pool, v_pool, page_table, seq_lens and
 *   workspace (and the *_dev buffers) are DEVICE pointers of the current
 *   CUDA device, 16-byte aligned, owned by the caller; *_host buffers are
 *   host memory.  The library never allocates or frees
 *   device memory and keeps no state between calls (re-entrant; the one
 *   exception, attn_decode_paged_noalloc, is described at its declaration).
 * - bf16 means IEEE bfloat16 stored in 16 bits; inputs are read as bf16,
 *   all arithmetic accumulates in fp32, outputs are rounded to bf16 with
 *   round-to-nearest-even.
 * - Calls are asynchronous on `stream` (NULL = legacy default stream).  The
 *   return value covers argument validation and the launch itself; a fault
 *   inside a kernel surfaces at the caller's next synchronisation.
 * - A zero-sized problem (B, N, Sq or Hq equal to 0) returns ATTN_OK and
 *   launches nothing.
 * - Masks.  With Sq query rows and Skv keys, off = Skv - Sq (bottom-right
 *   alignment).  Non-causal: every key is visible.  Causal: key j is visible
 *   to row i iff j <= i + off.  window W > 0 (causal only) additionally
 *   requires j > i + off - W: the query's own position and the W-1 before
 *   it.  A row with no visible key produces 0.
 * - GQA: query head h reads kv head h / (Hq / Hkv) (contiguous groups, the
 *   repeat_interleave order of the explainer's section 5.2); Hq must be a
 *   multiple of Hkv.  Hkv == Hq is MHA, Hkv == 1 is MQA.
 * - Device-side waits are bounded.  A kernel that gives up waiting, or that
 *   meets a page-table entry outside the pool, records it in a device error
 *   word and skips the affected work instead of faulting or hanging;
 *   attn_device_status() reads (and optionally clears) that word.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream; declared here so that callers
 * need no CUDA header. */
typedef struct CUstream_st* attn_stream_t;

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,   /* null pointer, negative size, Hq % Hkv != 0, misaligned pointer,
                                 attention head dim other than 64 or 128 */
  ATTN_ERR_UNSUPPORTED = 2,   /* valid but not implemented: page size, group size, window
                                 without causal, an append row size */
  ATTN_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed (launch, descriptor, device query) */
  ATTN_ERR_TIMEOUT = 4,       /* a device-side wait gave up (reported by attn_device_status) */
  ATTN_ERR_BAD_PAGE = 5,      /* a page-table entry was outside [0, num_pages), or a sequence was
                                 longer than max_pages * page_size or max_seq_len
                                 (reported by attn_device_status) */
  ATTN_ERR_WORKSPACE = 6,     /* workspace missing or smaller than attn_decode_paged_workspace_size */
  ATTN_ERR_OUT_OF_PAGES = 7   /* the page pool has too few free pages for a request (nothing changed) */
} attn_status_t;

/* Human-readable name of a status code (static string, never NULL). */
const char* attn_status_string(attn_status_t status);

/* Library version as 10000*major + 100*minor + patch. */
int attn_version(void);

/*
 * attn_prefill -- bf16 tiled prefill on the sm_100a tensor cores.
 *
 * q   : [B, Hq,  Sq,  D] bf16, contiguous (row-major, D innermost)
 * k, v: [B, Hkv, Skv, D] bf16, contiguous
 * out : [B, Hq,  Sq,  D] bf16, contiguous; must not alias q, k or v
 * D   : 64 or 128 (otherwise ATTN_ERR_INVALID_ARG)
 * scale : multiplier of q.k (1/sqrt(D) in the pages; passed explicitly)
 * causal: 0 or 1;  window: 0 = none, > 0 = sliding window (needs causal=1)
 *
 * Q.K^T and P.V run as tcgen05 MMAs (bf16 x bf16 -> fp32 in tensor memory)
 * on tiles staged by TMA; the softmax is the online form (running row max
 * and sum, accumulator rescaled when the max grows) and P is rounded to
 * bf16 before P.V.  Key tiles that the mask hides entirely are skipped.
 * Errors: ATTN_ERR_INVALID_ARG for null/misaligned pointers, bad sizes or D
 * not in {64,128}, ATTN_ERR_UNSUPPORTED for window>0 without causal,
 * ATTN_ERR_CUDA if the tensor-map encoder or the launch fails.
 */
attn_status_t attn_prefill(const void* q, const void* k, const void* v, void* out,
                           int B, int Hq, int Hkv, int Sq, int Skv, int D,
                           float scale, int causal, int window, attn_stream_t stream);

/*
 * attn_prefill_lse -- attn_prefill that also returns the log-sum-exp of every
 * query row ("Attention From Scratch" README, section "Quick start": the
 * Flash Attention module returns (output, lse)):
 *
 *     lse[b, h, i] = log( sum over visible j of exp(q_i . k_j * scale) )
 *
 * natural logarithm, fp32; -inf for a row with no visible key.  With it,
 * attention over two disjoint key sets can be merged exactly:
 * O = (e^lse1 O1 + e^lse2 O2) / (e^lse1 + e^lse2).
 * lse : [B, Hq, Sq] float, 4-byte aligned, device; must not be null.
 * Everything else as attn_prefill.
 */
attn_status_t attn_prefill_lse(const void* q, const void* k, const void* v, void* out, float* lse,
                               int B, int Hq, int Hkv, int Sq, int Skv, int D,
                               float scale, int causal, int window, attn_stream_t stream);

/*
 * attn_prefill_host -- attn_prefill whose inputs and output live in host
 * memory: the call copies q, k, v to the device, computes, and copies out
 * back, cutting the work into `chunks` pieces so that the two copy
 * directions and the kernels overlap.  A piece is a run of consecutive
 * (batch, kv head) pairs with their query heads; it is contiguous in every
 * buffer, so each of its transfers is a single copy, and its kernel is the
 * attn_prefill of those heads, with the same results bit for bit.
 *
 * q_host, k_host, v_host, out_host : host buffers with the layouts of
 *     attn_prefill.  Page-locked memory (cudaHostAlloc, cudaHostRegister)
 *     is needed for the copies to overlap anything; pageable memory gives
 *     the same results, copied synchronously.  The host must not touch
 *     out_host (nor change the inputs) until `stream` has completed.
 * q_dev, k_dev, v_dev, out_dev : device buffers of the same sizes, owned by
 *     the caller (the library allocates nothing), 16-byte aligned; their
 *     contents are overwritten.  k/v buffers may be null when Skv == 0.
 * chunks : pieces, 1 .. B * Hkv; 0 = one piece per 48 MB of input,
 *     rounded, at least two and at most eight (at most B * Hkv).  The host
 *     link bounds the call; more pieces shorten the last piece's kernel and
 *     copy back, which follow the last input copy, and each piece adds some
 *     copy and launch latency.
 * stream : the stream of the kernels.  When `stream` completes, every copy
 *     of the call has completed; the copies start only after work that was
 *     on `stream` before the call.
 * copy_in, copy_out : streams for the host-to-device and device-to-host
 *     copies, or NULL to use `stream` (no overlap).  For overlap they must
 *     be distinct from `stream` and from each other.
 * B, Hq, Hkv, Sq, Skv, D, scale, causal, window : as attn_prefill.
 * Errors: as attn_prefill (the device buffers take the place of q, k, v,
 * out in the checks); ATTN_ERR_INVALID_ARG for a null host buffer or chunks
 * out of range; ATTN_ERR_CUDA if a copy, event or launch call fails, in
 * which case the pieces enqueued before the failure stay enqueued and
 * `stream` still waits for their copies.
 */
attn_status_t attn_prefill_host(const void* q_host, const void* k_host, const void* v_host, void* out_host,
                                void* q_dev, void* k_dev, void* v_dev, void* out_dev,
                                int B, int Hq, int Hkv, int Sq, int Skv, int D,
                                float scale, int causal, int window, int chunks,
                                attn_stream_t stream, attn_stream_t copy_in, attn_stream_t copy_out);

/*
 * attn_prefill_f32 -- the same operation with fp32 inputs and output, fp32
 * arithmetic throughout (FFMA on the CUDA cores; no TF32), for results
 * that must agree with a float64 evaluation to about 1e-5.
 *
 * q : [B, Hq, Sq, D] float; k, v: [B, Hkv, Skv, D] float; out: [B, Hq, Sq, D] float.
 * D : 64 or 128.  Other arguments and errors as attn_prefill.
 */
attn_status_t attn_prefill_f32(const float* q, const float* k, const float* v, float* out,
                               int B, int Hq, int Hkv, int Sq, int Skv, int D,
                               float scale, int causal, int window, attn_stream_t stream);

/* attn_prefill_f32 with the per-row log-sum-exp, as attn_prefill_lse. */
attn_status_t attn_prefill_f32_lse(const float* q, const float* k, const float* v, float* out, float* lse,
                                   int B, int Hq, int Hkv, int Sq, int Skv, int D,
                                   float scale, int causal, int window, attn_stream_t stream);

/*
 * attn_prefill_paged -- bf16 prefill of a chunk of new tokens whose keys and
 * values sit in a paged KV cache (chunked prefill: the cache pages of the
 * "Attention From Scratch" README, section "Paged KV Cache", read by the
 * tiled prefill of attn_prefill).
 *
 * q          : [B, Hq, Sq, D] bf16, the queries of the Sq newest tokens of
 *              every sequence (the chunk being prefilled)
 * k_pool     : [num_pages, Hkv, page_size, D] bf16; v_pool the same
 * page_table : [B, max_pages] int32; entry p of row b holds tokens
 *              [p*page_size, (p+1)*page_size) of sequence b
 * seq_lens   : [B] int32 (device): tokens in each cache, the chunk's own
 *              included (its K/V already appended); query i of sequence b
 *              sits at position seq_lens[b] - Sq + i (bottom-right alignment)
 * page_size  : 16, 32, 64, 128 or 256
 * max_seq_len: host-side upper bound of seq_lens (longer sequences are
 *              truncated and reported as ATTN_ERR_BAD_PAGE by attn_device_status)
 * out        : [B, Hq, Sq, D] bf16;  lse: [B, Hq, Sq] float or NULL (as attn_prefill_lse)
 * causal / window / scale / D: as attn_prefill (causal = 0 lets every query see
 *              all seq_lens[b] keys).
 * Only the pages that hold a sequence's tokens are read; entries past its
 * last page are never read.  The slots of the last page after the final
 * token may hold anything, NaN included: they are masked, and their values
 * are cleared before they reach the output.  A page-table entry outside
 * [0, num_pages) for a token that the sequence holds is never read: it is
 * reported as ATTN_ERR_BAD_PAGE by attn_device_status and its keys
 * contribute garbage instead.
 * Errors: ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED, ATTN_ERR_CUDA.
 */
attn_status_t attn_prefill_paged(const void* q, const void* k_pool, const void* v_pool,
                                 const int32_t* page_table, const int32_t* seq_lens,
                                 int page_size, int B, int Hq, int Hkv, int Sq, int D,
                                 int num_pages, int max_pages, int max_seq_len,
                                 float scale, int causal, int window,
                                 void* out, float* lse, attn_stream_t stream);

/*
 * attn_decode_paged -- one decode step for N sequences over a paged KV cache.
 *
 * q          : [N, Hq, D] bf16, the new token's query of every sequence
 * k_pool     : [num_pages, Hkv, page_size, D] bf16, shared page pool
 * v_pool     : [num_pages, Hkv, page_size, D] bf16
 * page_table : [N, max_pages] int32; entry p of row b is the physical page
 *              holding tokens [p*page_size, (p+1)*page_size) of sequence b.
 *              Entries past a sequence's last page are never read.
 * seq_lens   : [N] int32 (device), tokens in each cache INCLUDING the new
 *              token (its k/v are already appended); 0 gives a zero output.
 * page_size  : tokens per page, a multiple of 16 in [16, 256]
 * max_seq_len: host-side upper bound of seq_lens, used only to size the
 *              split-KV grid; longer sequences are reported as
 *              ATTN_ERR_BAD_PAGE by attn_device_status and truncated.
 * window     : 0 = attend to all seq_lens[b] keys; W > 0 = the last W keys.
 * workspace  : device scratch of at least
 *              attn_decode_paged_workspace_size(N, Hq, D, max_seq_len, page_size)
 *              bytes, 16-byte aligned; the call uses it for the per-split
 *              partial outputs and log-sum-exps; contents are not needed
 *              between calls.  Two calls in flight at once need two
 *              workspaces.
 * out        : [N, Hq, D] bf16
 * D = 128 or 64; Hq / Hkv in {1, 2, 4, 8} (another group size gives
 * ATTN_ERR_UNSUPPORTED).
 *
 * Two kernels run on `stream`: a split-KV pass (one CTA per sequence, kv
 * head and span of keys; the query heads of a GQA group share every K/V
 * page read; pages are fetched whole by bulk asynchronous copies through
 * the page table) and a combine pass that merges the splits by their
 * log-sum-exp.  Errors: ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED,
 * ATTN_ERR_WORKSPACE, ATTN_ERR_CUDA.
 */
attn_status_t attn_decode_paged(const void* q, const void* k_pool, const void* v_pool,
                                const int32_t* page_table, const int32_t* seq_lens,
                                int page_size, int N, int Hq, int Hkv, int D,
                                int num_pages, int max_pages, int max_seq_len,
                                float scale, int window,
                                void* workspace, size_t workspace_bytes,
                                void* out, attn_stream_t stream);

/*
 * attn_decode_step_host -- one serving decode step whose per-step inputs and
 * output live in host memory ("Taking LLMs apart (2)", section "KV cache":
 * each step stores the new token's key and value in the cache, then attends
 * over the whole cache; "Attention From Scratch" README, section "Paged KV
 * Cache": the cache is a shared pool of pages).  On `stream`, in order:
 *   1. q_host -> q_dev, k_new_host -> k_new_dev, v_new_host -> v_new_dev;
 *   2. attn_kv_append of the new token (S_new = 1) at position
 *      seq_lens[b] - 1 of every sequence (seq_lens already counts it);
 *   3. attn_decode_paged over the pools into out_dev;
 *   4. out_dev -> out_host.
 * The cache (pools, page_table, seq_lens, workspace) stays on the device:
 * it is state, not per-step input.
 *
 * q_host, out_host : [N, Hq, D] bf16 host buffers; k_new_host, v_new_host :
 *     [N, Hkv, 1, D] bf16.  Page-locked memory is needed for the copies to
 *     run asynchronously; the host must not touch out_host, nor change the
 *     inputs, until `stream` has completed.
 * q_dev, out_dev : [N, Hq, D] bf16 device buffers; k_new_dev, v_new_dev :
 *     [N, Hkv, 1, D]; owned by the caller, 16-byte aligned, overwritten.
 * Other arguments : as attn_decode_paged (the pools are written by the
 *     append, so they are not const here).
 * Errors: as attn_kv_append and attn_decode_paged; ATTN_ERR_INVALID_ARG for a
 * null host or device buffer; ATTN_ERR_CUDA if a copy or launch fails (work
 * enqueued before the failure stays enqueued).
 */
attn_status_t attn_decode_step_host(const void* q_host, const void* k_new_host, const void* v_new_host,
                                    void* out_host, void* q_dev, void* k_new_dev, void* v_new_dev,
                                    void* out_dev, void* k_pool, void* v_pool,
                                    const int32_t* page_table, const int32_t* seq_lens,
                                    int page_size, int N, int Hq, int Hkv, int D,
                                    int num_pages, int max_pages, int max_seq_len,
                                    float scale, int window,
                                    void* workspace, size_t workspace_bytes,
                                    attn_stream_t stream);

/*
 * attn_decode_paged_noalloc -- attn_decode_paged for callers that cannot
 * allocate device memory: callers behind an interface with no workspace
 * argument (a plugin ABI fixed by a host framework), or serving loops whose
 * device memory is planned once at start-up, where a cudaMalloc (which may
 * also synchronise the device) is not allowed at decode time.  The source
 * pages have no counterpart; this is a deployment variant of the same call.
 *
 * Arguments, layouts and results are those of attn_decode_paged without the
 * workspace pair.  The split partials live in a fixed 32 MiB array inside
 * the library, which every GPU that loads the library holds until the
 * process exits; the call allocates and frees nothing.
 * - Sizes whose attn_decode_paged_workspace_size exceeds 32 MiB
 *   (33554432 bytes) are rejected with ATTN_ERR_WORKSPACE before any launch.
 * - The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.
 * - All calls share the array: calls that overlap on the GPU (other streams,
 *   other host threads) race on it and must be serialised by the caller.
 *   Nothing in it needs clearing between calls.
 * Errors: as attn_decode_paged, plus ATTN_ERR_WORKSPACE for sizes over the
 * limit and ATTN_ERR_CUDA if the address lookup fails.
 */
attn_status_t attn_decode_paged_noalloc(const void* q, const void* k_pool, const void* v_pool,
                                        const int32_t* page_table, const int32_t* seq_lens,
                                        int page_size, int N, int Hq, int Hkv, int D,
                                        int num_pages, int max_pages, int max_seq_len,
                                        float scale, int window, void* out, attn_stream_t stream);

/*
 * attn_decode_paged_fp8 -- attn_decode_paged over a cache stored as 8-bit
 * floats: k_pool and v_pool hold FP8 E4M3 codes (1 sign, 4 exponent bits with
 * bias 7, 3 mantissa bits, subnormals; no infinity; the codes 0x7F and 0xFF
 * are NaN), one byte per element, in the same [num_pages, Hkv, page_size, D]
 * layout.  An element stands for k_scale * e4m3(code) (v_scale for V):
 *     O = softmax((q . k_scale*K) * scale) (v_scale*V).
 * q and out stay bf16.  The pages give no 8-bit cache: this is a storage
 * variant of the decode above that halves the bytes it reads, with the same
 * arithmetic after the exact conversion of each code.
 * k_scale, v_scale: finite and > 0.  Every other argument, the workspace
 * (attn_decode_paged_workspace_size) and the errors are as attn_decode_paged.
 */
attn_status_t attn_decode_paged_fp8(const void* q, const uint8_t* k_pool, const uint8_t* v_pool,
                                    const int32_t* page_table, const int32_t* seq_lens,
                                    int page_size, int N, int Hq, int Hkv, int D,
                                    int num_pages, int max_pages, int max_seq_len,
                                    float scale, float k_scale, float v_scale, int window,
                                    void* workspace, size_t workspace_bytes, void* out, attn_stream_t stream);

/* Bytes of workspace attn_decode_paged needs for these sizes (0 if any size
 * is invalid).  Pure host arithmetic, no CUDA call. */
size_t attn_decode_paged_workspace_size(int N, int Hq, int D, int max_seq_len, int page_size);

/*
 * attn_device_status -- read the device error word of the current device
 * (synchronises the device).  Returns ATTN_OK if no kernel has recorded an
 * error since the last clear, ATTN_ERR_TIMEOUT if a bounded wait gave up,
 * ATTN_ERR_BAD_PAGE if a page-table entry or sequence length was out of
 * range, ATTN_ERR_CUDA if the read itself failed.  clear != 0 resets the word.
 */
attn_status_t attn_device_status(int clear);

/*
 * attn_selftest_wait_timeout -- exercise the failure path of the kernels'
 * bounded waits.  Launches one thread that waits, with the same wait the
 * kernels use, for an mbarrier phase that nothing completes; after limit_ms
 * milliseconds (1 to 1000) the wait gives up, records ATTN_ERR_TIMEOUT in
 * the device error word and the kernel returns.  attn_device_status then
 * reports ATTN_ERR_TIMEOUT, and the CUDA context stays usable.  A
 * diagnostic with no counterpart in the pages.
 * Errors: ATTN_ERR_INVALID_ARG (limit out of range), ATTN_ERR_CUDA.
 */
attn_status_t attn_selftest_wait_timeout(int limit_ms, attn_stream_t stream);

/*
 * ---------------------------------------------------------------------------
 * Paged KV cache management: a host-side page pool and the append kernel.
 *
 * The "Attention From Scratch" README (section "Paged KV Cache") splits the
 * cache into fixed-size pages held in one global pool, keeps a page table per
 * sequence, and allocates and reclaims pages as sequences grow and finish;
 * "LLM core technology" (section "PagedAttention") maps a sequence's logical
 * blocks to non-contiguous physical blocks through that table.  Its "KV
 * Cache" section, like the kv-cache walkthrough of "Taking LLMs apart (2)",
 * appends the new token's k and v to the cache before the attention of that
 * step.  The pool below manages the page ids and tables that attn_kv_append,
 * attn_prefill_paged and attn_decode_paged consume; the K/V pools themselves
 * are device memory the caller owns.
 * ---------------------------------------------------------------------------
 */

/* Opaque host object.  It holds a free list of page ids 0..num_pages-1 and,
 * for each sequence slot 0..max_seqs-1, its length in tokens and its page
 * list (the row of the page table).  Not thread-safe: callers serialise. */
typedef struct attn_page_pool attn_page_pool_t;

/*
 * attn_page_pool_create -- make a pool of num_pages pages of page_size tokens
 * for up to max_seqs sequences of at most max_pages_per_seq pages each.  All
 * pages start free and every sequence empty.  *pool receives the handle (host
 * memory allocated by the library, released by attn_page_pool_destroy).
 * Errors: ATTN_ERR_INVALID_ARG for a null handle pointer or a size <= 0.
 */
attn_status_t attn_page_pool_create(int num_pages, int page_size, int max_seqs, int max_pages_per_seq,
                                    attn_page_pool_t** pool);

/* Free the pool's host memory (NULL is a no-op).  Device copies made by
 * attn_page_pool_upload are the caller's and stay valid. */
void attn_page_pool_destroy(attn_page_pool_t* pool);

/*
 * attn_page_pool_resize -- set sequence `seq` to `len` tokens.  Growing takes
 * ceil(len / page_size) - (pages held) pages from the free list and appends
 * them to the sequence's page list; shrinking returns the pages past
 * ceil(len / page_size) to the free list (the most recently freed page is
 * the next one handed out).  Tokens already in the kept pages do not move.
 * All or nothing: with too few free pages the call returns
 * ATTN_ERR_OUT_OF_PAGES and changes nothing.
 * Errors: ATTN_ERR_INVALID_ARG (null pool, seq out of range, len < 0 or
 * more than max_pages_per_seq * page_size), ATTN_ERR_OUT_OF_PAGES.
 */
attn_status_t attn_page_pool_resize(attn_page_pool_t* pool, int seq, int len);

/* attn_page_pool_release -- end sequence `seq`: all its pages go back to the
 * free list and its length becomes 0 (resize to 0). */
attn_status_t attn_page_pool_release(attn_page_pool_t* pool, int seq);

/* Free pages left in the pool (-1 for a null pool). */
int attn_page_pool_free_pages(const attn_page_pool_t* pool);

/* Length in tokens of sequence `seq` (-1 for a null pool or seq out of range). */
int attn_page_pool_seq_len(const attn_page_pool_t* pool, int seq);

/*
 * attn_page_pool_export -- copy the pool's state to HOST arrays:
 * page_table [max_seqs, max_pages_per_seq] int32 (row s = the page ids of
 * sequence s in token order, -1 after its last page) and seq_lens [max_seqs]
 * int32.  Either pointer may be NULL to skip it.
 */
attn_status_t attn_page_pool_export(const attn_page_pool_t* pool, int32_t* page_table, int32_t* seq_lens);

/*
 * attn_page_pool_upload -- copy the rows changed since the last upload to the
 * DEVICE arrays page_table [max_seqs, max_pages_per_seq] and seq_lens
 * [max_seqs] (int32, laid out as attn_page_pool_export), with
 * cudaMemcpyAsync on `stream`.  The first upload copies everything.  The
 * copies read the pool's own pageable host memory, which the CUDA runtime
 * stages before the call returns, so the pool may be changed right after.
 * Kernels later on `stream` see the new tables.
 * Errors: ATTN_ERR_INVALID_ARG (null pointer), ATTN_ERR_CUDA.
 */
attn_status_t attn_page_pool_upload(attn_page_pool_t* pool, int32_t* page_table, int32_t* seq_lens,
                                    attn_stream_t stream);

/*
 * attn_kv_append -- write the keys and values of S_new new tokens of each of
 * B sequences into the paged cache.
 *
 * k_new, v_new : [B, Hkv, S_new, D] bf16 (the k/v layout of attn_prefill;
 *                one decode step is S_new = 1)
 * k_pool, v_pool: [num_pages, Hkv, page_size, D] bf16, written in place
 * page_table   : [B, max_pages] int32 (device)
 * seq_lens     : [B] int32 (device), the cache lengths AFTER the append (the
 *                array that attn_prefill_paged / attn_decode_paged then take):
 *                token i of sequence b goes to position seq_lens[b] - S_new + i,
 *                i.e. page page_table[b][pos / page_size], slot pos % page_size.
 *                Positions below 0 (a cache shorter than the chunk) are skipped.
 * page_size    : a multiple of 8 tokens; D a multiple of 8, at most 512.
 * A position past max_pages * page_size, or a page-table entry outside
 * [0, num_pages), writes nothing and is reported as ATTN_ERR_BAD_PAGE by
 * attn_device_status.  The values are copied bit for bit.
 * Errors: ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED, ATTN_ERR_CUDA.
 */
attn_status_t attn_kv_append(const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                             const int32_t* page_table, const int32_t* seq_lens,
                             int page_size, int B, int Hkv, int S_new, int D,
                             int num_pages, int max_pages, attn_stream_t stream);

/*
 * attn_kv_append_fp8 -- attn_kv_append into an 8-bit cache (the pools of
 * attn_decode_paged_fp8).  Each bf16 element x of k_new (v_new) becomes the
 * E4M3 code nearest to x * (1 / k_scale) (v_scale): the reciprocal and the
 * product are rounded to float32, the code to nearest with ties to the even
 * code, and magnitudes above 448 saturate to +-448 (cvt.rn.satfinite).
 * k_pool, v_pool: [num_pages, Hkv, page_size, D] uint8.  k_scale, v_scale:
 * finite and > 0.  Everything else, the errors included, is as attn_kv_append.
 */
attn_status_t attn_kv_append_fp8(const void* k_new, const void* v_new, uint8_t* k_pool, uint8_t* v_pool,
                                 const int32_t* page_table, const int32_t* seq_lens,
                                 int page_size, int B, int Hkv, int S_new, int D,
                                 int num_pages, int max_pages, float k_scale, float v_scale,
                                 attn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */

/*
 * infllmv2.h -- C ABI of libinfllmv2.so: the InfLLM v2 sparse-attention path on NVIDIA B200 (sm_100a).
 *
 * The method (MiniCPM4 pages; cited by page title and section):
 *   (1) semantic kernels: every KV head's key cache is summarised by "fine-grained semantic kernels",
 *       here the mean of K over a 32-key window advanced by 16 keys;
 *   (2) a query token's relevance to a 64-key context block is the max over the block's kernels of the
 *       query-kernel score; the query heads of one GQA group share one block set; the top-k blocks are
 *       taken, together with the initial block and the local blocks;
 *   (3) attention runs over the selected blocks only, causally, for prefill and decode, with dense
 *       attention for short contexts.
 *   Sources: "Tsinghua & ModelBest: MiniCPM4 technical details" (QbitAI), section "Model architecture:
 *   InfLLM v2", items 1) finer semantic kernels, 2) GQA-group query-head sharing, 3) operators and the
 *   LogSumExp-based top-k; "MiniCPM 4.0 launch article" (senqingzn.com), section 1 "efficient
 *   architecture" (dense/sparse switch); QbitAI article, section "speculative sampling, quantisation
 *   and long text", long-context bullet (tree-draft verification with a bit-packed local mask).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library allocates no device memory.
 *     Between calls it keeps only: per-device caches of kernel attributes and cluster occupancy, the
 *     device-side flags that bounded waits raise (read and cleared by infllmv2_device_status), and the
 *     fixed scratch array of infllmv2_sparse_attn_decode_noalloc.  Every call is asynchronous on `stream`
 *     (0 = legacy default stream).
 *   - bf16 = IEEE bfloat16 (2 bytes).  Layouts are dense row-major (innermost index last):
 *       q        [B, T, Hq, d]       queries (T query tokens per sequence)
 *       k, v     [B, Lcap, Hkv, d]   key / value cache, position-major
 *       kern     [B, Hkv, nk_cap, d] semantic-kernel cache, bf16
 *       idx      [B, T, Hkv, kmax]   int32 selected block ids, ascending, -1 padded; kmax = topk +
 *                                    init_blocks + local_blocks
 *       cnt      [B, T, Hkv]         int32 number of selected blocks
 *       out      [B, T, Hq, d]       bf16; lse [B, T, Hq] fp32 natural-log softmax denominator (nullable)
 *     GQA: query head h reads KV head h / (Hq / Hkv).
 *   - Context of a query: n = the number of cache keys it may see.  q_ctx[b*T + t] gives it; when q_ctx
 *     is NULL the T queries are the last T tokens of a causal sequence: n = ctx_lens[b] - T + t + 1.
 *     Kernels visible to the query are the complete windows inside [0, n); its own block is c = (n-1)/64.
 *   - Dense switch: a query with n <= params.dense_len attends to all keys [0, n).  Its selection row is
 *     written as cnt = c + 1 with the first min(c + 1, kmax) block ids; attention ignores idx for it.
 *   - Pointers must be 16-byte aligned; d must be 64 or 128; Hq / Hkv in {1, 2, 4, 8, 16}; the GPU path
 *     supports block_size 64, kernel_size 32, kernel_stride 16 (other values -> INFLLMV2_ERR_UNSUPPORTED).
 *   - Errors: every argument is checked on the host before any launch; on a bad argument the call
 *     returns the status and launches nothing.  A failed launch returns INFLLMV2_ERR_CUDA.  Kernels
 *     never wait on other kernels or devices; waits inside one CTA are bounded (infllmv2_device_status).
 *   - Workspace: entry points that take (ws, ws_bytes) need at least infllmv2_workspace_size(...) bytes
 *     of device memory, 256-byte aligned, owned by the caller; calls that run concurrently need separate
 *     workspaces.  Its contents need no initialisation and are scratch after the call.
 */
#ifndef INFLLMV2_H
#define INFLLMV2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* infllmv2_stream_t; /* same type as cudaStream_t */

typedef enum {
    INFLLMV2_OK = 0,
    INFLLMV2_ERR_INVALID_ARG = 1, /* null/misaligned pointer, negative or inconsistent size */
    INFLLMV2_ERR_UNSUPPORTED = 2, /* valid but outside what the GPU kernels implement */
    INFLLMV2_ERR_WORKSPACE = 3,   /* workspace missing, misaligned or too small */
    INFLLMV2_ERR_CUDA = 4,        /* a CUDA launch failed (cudaGetLastError after the launch) */
    INFLLMV2_ERR_TIMEOUT = 5      /* a bounded device-side wait ran out (see infllmv2_device_status) */
} infllmv2_status;

/* Method constants (the pages give none; the workloads use 64 / 32 / 16, k = 8 or 64, 1 + 2 forced). */
typedef struct {
    int block_size;      /* keys per context block (GPU: 64) */
    int kernel_size;     /* keys per semantic-kernel window (GPU: 32) */
    int kernel_stride;   /* stride between windows (GPU: 16) */
    int topk;            /* blocks chosen by score besides the forced ones, 0 <= topk <= 2^24 */
    int init_blocks;     /* blocks [0, init_blocks) always kept, 0 <= init_blocks <= 2^24 */
    int local_blocks;    /* the query's own block and the local_blocks-1 before it always kept, 0 .. 2^24 */
    int dense_len;       /* queries with context n <= dense_len attend densely */
    int membership;      /* 0 = OVERLAP: kernel j belongs to every block its window intersects;
                            1 = CONTAINED: only to the block that contains its whole window */
    float softmax_scale; /* <= 0 selects 1/sqrt(d); used for kernel scoring and attention */
    int lse_stride;      /* 0 or 1: exact LSE_h.  2, 4 or 8: the estimate LSE_h ~ log(s * sum of exp z_h(j) over the
                            visible kernels j = 0, s, 2s, ...), one reading of the LogSumExp estimation the pages
                            name for fast top-k (QbitAI, "Model architecture: InfLLM v2", item 3; the pages do
                            not define it).  Only the prefill scoring on the tensor cores (16 heads per group,
                            d 128) takes it; other scoring paths return INFLLMV2_ERR_UNSUPPORTED */
} infllmv2_params;

/* Human-readable name of a status code (static storage). */
const char* infllmv2_status_string(int status);

/* Library version, as major*10000 + minor*100 + patch. */
int infllmv2_version(void);

/*
 * Device-side status of the kernels that wait on their own producer/consumer barriers (the tensor-core
 * prefill scoring and attention, the one-launch decode step): every such wait is bounded, and a wait that
 * runs out records an error, makes its CTA skip the rest of its work and exit.  Returns INFLLMV2_ERR_TIMEOUT if that happened since the last
 * call (and clears the record), INFLLMV2_OK otherwise, INFLLMV2_ERR_CUDA if the record cannot be read.
 * Synchronous: it reads device memory on the current device.
 */
int infllmv2_device_status(void);

/*
 * Testing only (the pages have no counterpart): with polls > 0, the first kernel-cache wait of every CTA of
 * the fused decode step (infllmv2_sparse_decode_step and its paged form) polls a barrier that nothing
 * arrives on and gives up after `polls` polls, as a wait whose copy never lands would after its normal
 * limit.  That drives the bounded-wait error path without a fault: the step's CTAs issue no further copy,
 * wait (bounded) for the copies in flight, still reach every cluster barrier, and infllmv2_device_status then
 * returns INFLLMV2_ERR_TIMEOUT; the step's outputs are not the method's.  The same limit applies to the
 * first wait of the MMA-issuing thread in every CTA of the tensor-core prefill kernels: the attention
 * (infllmv2_sparse_attn_prefill, its paged and packed forms) and the scoring with top-k
 * (infllmv2_block_score_topk and its packed form), on their tcgen05 paths.  Their CTAs then stop their loops;
 * each producer waits (bounded) for the copies it issued, and each MMA issuer for its MMAs.  The CTAs free
 * their TMEM and exit, and infllmv2_device_status returns INFLLMV2_ERR_TIMEOUT; idx / cnt or the attention
 * outputs of that call are not the method's.  polls = 0 restores the normal waits.  The limit is process-wide and becomes a launch argument of every such kernel launched after
 * this returns (a CUDA graph captured before keeps the value it captured).  Returns INFLLMV2_OK.
 */
int infllmv2_test_set_first_wait_limit(unsigned polls);

/*
 * Bytes of workspace the calls below need for problems up to the given sizes (host-only, no CUDA call).
 *   max_q   : largest T (queries per sequence) of any call
 *   max_ctx : largest context length n of any query
 * Returns 0 when the arguments are invalid.
 */
size_t infllmv2_workspace_size(const infllmv2_params* params, int batch, int max_q, int max_ctx, int hq, int hkv,
                               int head_dim);

/*
 * Cache maintenance of a decode step (the pages have no counterpart; it keeps a step's host traffic to one
 * copy of the new rows): writes one new key and one new value row per sequence into the caches,
 *   k_cache[b, pos[b], :, :] = k_new[b, :, :]   and   v_cache[b, pos[b], :, :] = v_new[b, :, :]
 *   k_new, v_new      [B, Hkv, d] bf16 (device, 16-byte aligned)
 *   pos               [B] int32 (device); a position outside [0, Lcap) writes nothing
 *   k_cache, v_cache  [B, Lcap, Hkv, d] bf16 (device, 16-byte aligned); rows other than pos[b] untouched
 * Ordered on `stream` like every call here; the new rows are visible to the calls enqueued after it.
 */
int infllmv2_kv_append(const void* k_new, const void* v_new, int batch, int hkv, int head_dim, const int32_t* pos,
                       void* k_cache, void* v_cache, int lcap, infllmv2_stream_t stream);

/*
 * Step 1 -- semantic kernels (MiniCPM4 technical details, "Model architecture: InfLLM v2", item 1).
 * For each sequence b, writes the kernels completed between old_lens[b] and new_lens[b] keys:
 *   kern[b, g, j, :] = bf16_round_nearest_even( mean_{i in [16 j, 16 j + 32)} k[b, i, g, :] )
 * for j in [nk(old), nk(new)), nk(n) = n >= 32 ? (n - 32) / 16 + 1 : 0.  The window sum is formed in fp64
 * (exact unless the 32 keys' exponents spread over more than ~40 binary orders) and the mean is rounded once
 * to bf16, so the result is the correctly rounded mean.
 *   k            [B, Lcap, Hkv, d] bf16 (device)
 *   old_lens,
 *   new_lens     [B] int32 (device), 0 <= old <= new <= Lcap; device-side values are trusted
 *   max_new_keys host upper bound of new_lens[b] - old_lens[b] over b (sizes the grid; 1 for a decode
 *                step, the prompt length for a prefill)
 *   kern         [B, Hkv, nk_cap, d] bf16 (device); requires nk(new_lens[b]) <= nk_cap
 */
int infllmv2_kernel_pool(const void* k, int batch, int lcap, int hkv, int head_dim, const int32_t* old_lens,
                         const int32_t* new_lens, int max_new_keys, const infllmv2_params* params, void* kern,
                         int nk_cap, infllmv2_stream_t stream);

/*
 * Backward of step 1 (training: MiniCPM4 technical details, "Model architecture: InfLLM v2", item 3 -- the
 * operators serve training as well as inference; the pages give no formula, so this is the derivative of step
 * 1's definition, with the bf16 rounding of the kernels taken as the identity).  For a loss that depends on the
 * kernels differentiably (the attention backward passes no gradient through them), the transpose of the
 * window mean:
 *   dk[b, i, g, :] (+)= sum_{j < nk(lens[b]), 16 j <= i < 16 j + 32} dkern[b, g, j, :] / 32,  i in [0, lens[b])
 * i.e. each key of the 16-key chunk c gets (dkern[c - 1] + dkern[c]) / 32, a term only for a complete window.
 * The pair is summed in fp32 with one rounding and scaled exactly, so with accumulate = 0 a normal result is
 * the correctly rounded exact value.
 *   dkern      [B, Hkv, nk_cap, d] fp32 (device, 16-byte aligned)
 *   lens       [B] int32 (device): keys per sequence; values past lcap are clamped to it, kernels past nk_cap
 *              are not read
 *   max_len    host upper bound of lens[b] (sizes the grid): 0 <= max_len <= lcap, nk(max_len) <= nk_cap
 *   dk         [B, Lcap, Hkv, d] fp32 (device, 16-byte aligned).  accumulate = 1 adds into rows [0, lens[b])
 *              (e.g. onto infllmv2_sparse_attn_backward's dk), 0 overwrites them; rows past lens[b] untouched.
 * B * Hkv <= 65535.  Returns INFLLMV2_OK, INFLLMV2_ERR_INVALID_ARG, INFLLMV2_ERR_UNSUPPORTED or
 * INFLLMV2_ERR_CUDA.
 */
int infllmv2_kernel_pool_backward(const float* dkern, int batch, int lcap, int hkv, int head_dim, const int32_t* lens,
                                  int max_len, const infllmv2_params* params, int nk_cap, float* dk, int accumulate,
                                  infllmv2_stream_t stream);

/*
 * Step 2 -- block scoring and top-k selection (same section, items 1-3).
 * For each query (b, t) and KV group g, with kernel scores z_h(j) = scale * q_h . kern_j over the visible
 * kernels and LSE_h = log sum_j exp z_h(j) (exact), the group score of block blk is
 *   S_g(blk) = sum_{h in g} max_{j in blk, visible} exp(z_h(j) - LSE_h)
 * (kernel j is in blk per params.membership).  Forced blocks [0, init) and [c - local + 1, c] are kept;
 * of the other blocks with a visible kernel, the topk with the largest S are taken (ties -> lower id).
 * The union is written ascending to idx[b, t, g, :], padded with -1, its size to cnt[b, t, g].
 *   q          [B, T, Hq, d] bf16 (device)
 *   q_ctx      [B * T] int32 (device) or NULL (then the T queries end the sequence: see above)
 *   ctx_lens   [B] int32 (device); required when q_ctx is NULL, else ignored (may be NULL)
 *   max_ctx    host upper bound of every query's n (sizes the grid and the workspace)
 *   kern       [B, Hkv, nk_cap, d] bf16 (device), valid for every kernel visible to the queries
 *   idx, cnt   outputs as described; kmax = topk + init_blocks + local_blocks
 *   ws         workspace of ws_bytes >= infllmv2_workspace_size(params, B, T, max_ctx, Hq, Hkv, d)
 */
int infllmv2_block_score_topk(const void* q, int batch, int num_q, int hq, int hkv, int head_dim,
                              const int32_t* q_ctx, const int32_t* ctx_lens, int max_ctx, const void* kern,
                              int nk_cap, const infllmv2_params* params, int32_t* idx, int32_t* cnt, void* ws,
                              size_t ws_bytes, infllmv2_stream_t stream);

/*
 * Step 3a -- block-sparse attention of T query tokens per sequence (prefill / chunked prefill)
 * (MiniCPM4 technical details, InfLLM v2 overview: only the selected blocks take part in attention).
 * Query (b, t), head h, group g = h / (Hq/Hkv), context n:
 *   keys = [0, n) if n <= dense_len, else the union over blk in idx[b, t, g, :cnt] of [64 blk, min(64 blk + 64, n))
 *   out[b, t, h, :] = sum_{i in keys} softmax_i(scale * q . k_i) v_i ; lse = log sum_i exp(scale * q . k_i)
 * Block ids must be ascending, unique, >= 0 and have 64 blk < n (checked on the device: an invalid id is
 * skipped).  k, v: [B, Lcap, Hkv, d] bf16.  lse may be NULL.  ws as for block_score_topk.
 */
int infllmv2_sparse_attn_prefill(const void* q, int batch, int num_q, int hq, int hkv, int head_dim, const void* k,
                                 const void* v, int lcap, const int32_t* q_ctx, const int32_t* ctx_lens,
                                 int max_ctx, const int32_t* idx, const int32_t* cnt,
                                 const infllmv2_params* params, void* out, float* lse, void* ws, size_t ws_bytes,
                                 infllmv2_stream_t stream);

/*
 * Step 3b -- block-sparse attention of one new token per sequence (decode; MiniCPM4 technical details,
 * efficiency evaluation: the number of blocks read stays constant as the context grows).  Same formula
 * as 3a with T = 1 and n = ctx_lens[b] (the new token's key and value are already in the cache).
 * Split over the selected blocks across CTAs, partial results merged by their LSE in the workspace.
 *   q [B, 1, Hq, d]; out [B, 1, Hq, d]; lse [B, Hq] or NULL.
 */
int infllmv2_sparse_attn_decode(const void* q, int batch, int hq, int hkv, int head_dim, const void* k,
                                const void* v, int lcap, const int32_t* ctx_lens, int max_ctx, const int32_t* idx,
                                const int32_t* cnt, const infllmv2_params* params, void* out, float* lse, void* ws,
                                size_t ws_bytes, infllmv2_stream_t stream);

/*
 * Steps 2 + 3b fused -- one decode step: block scoring, top-k selection and sparse attention of one new
 * token per sequence in a single launch, with no workspace (efficiency evaluation of the QbitAI article:
 * a decode step reads a constant number of blocks plus the kernel representations).  Writes exactly what
 * infllmv2_block_score_topk followed by infllmv2_sparse_attn_decode write (idx, cnt, out, lse) for the
 * same inputs: q [B, 1, Hq, d], n = ctx_lens[b], kernels visible up to n.  One thread-block cluster per
 * (sequence, KV group) scans the kernel cache, merges the per-head LSE partials and the block scores
 * over distributed shared memory, selects, and attends to the selected blocks.
 *   kern [B, Hkv, nk_cap, d]: the kernel cache, already pooled up to ctx_lens (infllmv2_kernel_pool).
 *   Limits: contexts up to 256K keys; B * Hkv <= 65535.
 */
int infllmv2_sparse_decode_step(const void* q, int batch, int hq, int hkv, int head_dim, const void* kern, int nk_cap,
                                const void* k, const void* v, int lcap, const int32_t* ctx_lens, int max_ctx,
                                const infllmv2_params* params, int32_t* idx, int32_t* cnt, void* out, float* lse,
                                infllmv2_stream_t stream);

/*
 * Steps 1 + 2 + 3b of one decode step in a single launch: infllmv2_kernel_pool of each sequence's last key
 * (old = n - 1, new = n keys, n = ctx_lens[b]) followed by infllmv2_sparse_decode_step, with the same results
 * (the kernel the last key completes, if it completes one, is written to kern bit for bit as the pooling call
 * writes it).  The CTA that scans that kernel's block pools it, from the 32 keys of its window in k, and uses it
 * in its scan.  Arguments as infllmv2_sparse_decode_step; kern is read and written, and must hold every kernel
 * of the first n - 1 keys.  q [B, 1, Hq, d].
 */
int infllmv2_sparse_decode_step_pool(const void* q, int batch, int hq, int hkv, int head_dim, void* kern, int nk_cap,
                                const void* k, const void* v, int lcap, const int32_t* ctx_lens, int max_ctx,
                                const infllmv2_params* params, int32_t* idx, int32_t* cnt, void* out, float* lse,
                                infllmv2_stream_t stream);

/*
 * Paged key/value cache (serving; the pages give no cache layout -- the CPM.cu runtime of the QbitAI
 * article, section "CPM.cu", manages static device memory, and a pool of fixed-size pages is that idea for
 * many sequences of unknown length).  One page holds one context block, 64 positions, so a selected block
 * is one page.  Position i of sequence b lives in row
 *     page_table[b * max_pages + i / 64] * 64 + i % 64
 * of the page pools k_pages / v_pages [num_pages * 64, Hkv, d] bf16 (device, 16-byte aligned).
 *   page_table   [B, max_pages] int32 (device, 4-byte aligned), owned by the caller; entries past a
 *                sequence's length are not read.  An entry outside [0, num_pages) is never dereferenced:
 *                its positions read as zeros and are not written (such a row's results are then not the
 *                method's; the Python binding's INFLLMV2_CHECK=1 mode checks the table on the host).
 *   1 <= num_pages <= 2^24 and 1 <= max_pages <= 4096 (contexts up to 256K positions), else
 *   INFLLMV2_ERR_UNSUPPORTED / INFLLMV2_ERR_INVALID_ARG.
 * Each call computes exactly its contiguous counterpart on the cache gathered through the page table:
 *   infllmv2_kv_append_paged          = infllmv2_kv_append        (writes through the table)
 *   infllmv2_kernel_pool_paged        = infllmv2_kernel_pool
 *   infllmv2_sparse_decode_step_paged = infllmv2_sparse_decode_step
 *   infllmv2_sparse_attn_prefill_paged = infllmv2_sparse_attn_prefill (chunked prefill: q holds the last T
 *                                      positions of each context; score them with infllmv2_block_score_topk,
 *                                      which reads only the kernel cache)
 * The kernel cache kern [B, Hkv, nk_cap, d] stays contiguous per sequence (1/16 of the keys).
 */
int infllmv2_kv_append_paged(const void* k_new, const void* v_new, int batch, int hkv, int head_dim, const int32_t* pos,
                             void* k_pages, void* v_pages, int num_pages, const int32_t* page_table, int max_pages,
                             infllmv2_stream_t stream);
int infllmv2_kernel_pool_paged(const void* k_pages, int num_pages, const int32_t* page_table, int max_pages,
                               int batch, int hkv, int head_dim, const int32_t* old_lens, const int32_t* new_lens,
                               int max_new_keys, const infllmv2_params* params, void* kern, int nk_cap,
                               infllmv2_stream_t stream);
int infllmv2_sparse_decode_step_paged(const void* q, int batch, int hq, int hkv, int head_dim, const void* kern,
                                      int nk_cap, const void* k_pages, const void* v_pages, int num_pages,
                                      const int32_t* page_table, int max_pages, const int32_t* ctx_lens, int max_ctx,
                                      const infllmv2_params* params, int32_t* idx, int32_t* cnt, void* out,
                                      float* lse, infllmv2_stream_t stream);
int infllmv2_sparse_attn_prefill_paged(const void* q, int batch, int num_q, int hq, int hkv, int head_dim,
                                       const void* k_pages, const void* v_pages, int num_pages,
                                       const int32_t* page_table, int max_pages, const int32_t* q_ctx,
                                       const int32_t* ctx_lens, int max_ctx, const int32_t* idx, const int32_t* cnt,
                                       const infllmv2_params* params, void* out, float* lse,
                                       infllmv2_stream_t stream);

/*
 * Steps 1 + 2 + 3a for a packed batch of variable-length sequences (serving prefill without padding; the
 * pages define no batching, this is the usual cu_seqlens packing).  Sequence b owns query rows
 * [cu_seqlens_q[b], cu_seqlens_q[b+1]) and key / value rows [cu_seqlens_k[b], cu_seqlens_k[b+1]); its
 * T_b queries are the last T_b of its L_b keys (query t sees n = L_b - T_b + t + 1 keys).  Three launches
 * for the whole batch: the kernel pool of every sequence's keys into kern[b], block scoring + top-k of
 * every query, and sparse attention -- per sequence exactly infllmv2_kernel_pool, infllmv2_block_score_topk
 * and infllmv2_sparse_attn_prefill on that sequence alone.
 *   q, out        [total_q, Hq, d] bf16;   k, v [total_k, Hkv, d] bf16
 *   cu_seqlens_q,
 *   cu_seqlens_k  [B + 1] int32 (device): 0 = cu[0] <= cu[1] <= ... , cu[B] = total; T_b <= L_b (trusted:
 *                 the Python binding checks them on the host under INFLLMV2_CHECK=1)
 *   max_seqlen_q, max_seqlen_k: host upper bounds of T_b and L_b (they size the grids)
 *   kern          [B, Hkv, nk_cap, d] bf16 (device), nk_cap >= the kernel count of max_seqlen_k; written
 *   idx, cnt      [total_q, Hkv, kmax] / [total_q, Hkv] int32;   lse [total_q, Hq] fp32 or NULL
 *   ws            >= infllmv2_workspace_size(params, B, max_seqlen_q, max_seqlen_k, Hq, Hkv, d) bytes
 */
int infllmv2_sparse_prefill_varlen(const void* q, const void* k, const void* v, int batch, int hq, int hkv, int head_dim,
                                   const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int total_q, int total_k,
                                   int max_seqlen_q, int max_seqlen_k, const infllmv2_params* params, void* kern,
                                   int nk_cap, int32_t* idx, int32_t* cnt, void* out, float* lse, void* ws,
                                   size_t ws_bytes, infllmv2_stream_t stream);

/*
 * Step 3c -- tree-draft verification (QbitAI article, "speculative sampling, quantisation and long text",
 * long-context bullet).  n_draft draft tokens per sequence, each a query that sees the whole prefix of
 * prefix_lens[b] cache keys through its own selected blocks (its q_ctx is the prefix length), plus the
 * draft tokens j whose bit j is set in tree_mask[b * n_draft + i] (its ancestors and itself):
 *   keys(i) = prefix keys of idx[b, i, g, :cnt] (clipped to the prefix, or all of it when
 *             prefix <= dense_len)  U  { draft j : bit j of tree_mask[b, i] }
 *   q [B, n_draft, Hq, d]; k_draft, v_draft [B, n_draft, Hkv, d] bf16; tree_mask [B, n_draft] uint32;
 *   n_draft <= 32; out [B, n_draft, Hq, d]; lse [B, n_draft, Hq] or NULL.
 */
int infllmv2_sparse_attn_tree_verify(const void* q, int batch, int n_draft, int hq, int hkv, int head_dim,
                                     const void* k, const void* v, int lcap, const int32_t* prefix_lens, int max_ctx,
                                     const void* k_draft, const void* v_draft, const uint32_t* tree_mask,
                                     const int32_t* idx, const int32_t* cnt, const infllmv2_params* params,
                                     void* out, float* lse, void* ws, size_t ws_bytes, infllmv2_stream_t stream);

/*
 * Sparse decode attention without a workspace.  The pages have no counterpart: this is a convenience of
 * the library.  It computes exactly what infllmv2_sparse_attn_decode computes, with the same arguments and
 * layouts minus (ws, ws_bytes), for callers that cannot allocate device memory when they call: a process
 * that hands out its GPU memory once at start-up, a plugin that may not use its host's allocator, a loop
 * that must never allocate.  The split partials go to a 4 MiB array inside the library instead (one per
 * GPU that loads the library, kept until the process exits).
 *   Limit: B * Hkv * ceil(max(kmax, blocks of min(max_ctx, dense_len)) / 4) * (16 * d + 32) * 4 bytes must
 *   fit in 4 MiB (for example B = 4, Hkv = 2, d = 128, kmax = 67, dense_len = 8192 needs 2.1 MiB); a larger
 *   call returns INFLLMV2_ERR_WORKSPACE and launches nothing.
 *   The first call on a device looks up the array's address (cudaGetSymbolAddress) with that device
 *   current; make it before any stream capture.  All calls share the array, so calls whose kernels overlap
 *   on the GPU (other streams or host threads) race on it.  Nothing in it needs clearing between calls.
 */
int infllmv2_sparse_attn_decode_noalloc(const void* q, int batch, int hq, int hkv, int head_dim, const void* k,
                                        const void* v, int lcap, const int32_t* ctx_lens, int max_ctx,
                                        const int32_t* idx, const int32_t* cnt, const infllmv2_params* params,
                                        void* out, float* lse, infllmv2_stream_t stream);

/*
 * Dense path (MiniCPM 4.0 launch article, section 1: short texts keep dense attention).  Plain causal GQA
 * attention over keys [0, n) for every query, whatever dense_len is; same layouts and n rules as 3a / 3b.
 */
int infllmv2_dense_attn_prefill(const void* q, int batch, int num_q, int hq, int hkv, int head_dim, const void* k,
                                const void* v, int lcap, const int32_t* q_ctx, const int32_t* ctx_lens, int max_ctx,
                                float softmax_scale, void* out, float* lse, void* ws, size_t ws_bytes,
                                infllmv2_stream_t stream);
int infllmv2_dense_attn_decode(const void* q, int batch, int hq, int hkv, int head_dim, const void* k, const void* v,
                               int lcap, const int32_t* ctx_lens, int max_ctx, float softmax_scale, void* out,
                               float* lse, void* ws, size_t ws_bytes, infllmv2_stream_t stream);

/*
 * Backward of step 3a for a fixed selection (training: MiniCPM4 technical details, "Model architecture:
 * InfLLM v2", item 3 -- the operators serve training as well as inference; the pages give no formula, so
 * this is the derivative of 3a's definition).  The selection is piecewise constant in q and K, so no
 * gradient flows through the block scores or the semantic kernels.  With the forward's key sets (3a) and
 * p_i = exp(scale q.k_i - lse), for a loss L with dout = dL/dout:
 *   dv_i += p_i dout;   ds_i = p_i (dout . v_i - dout . out);   dq = scale sum_i ds_i k_i;   dk_i += scale ds_i q
 * summed over every (query, head) that reads key i (GQA: the heads of a group add into one KV head).
 *   q, k, v, q_ctx, ctx_lens, max_ctx, idx, cnt, params: exactly as given to infllmv2_sparse_attn_prefill.
 *               idx and cnt both NULL: every query attends to all of [0, n) (the dense attention's backward).
 *   out        [B, T, Hq, d] bf16: the forward's output;  lse [B, T, Hq] fp32: the forward's lse (required)
 *   dout       [B, T, Hq, d] bf16
 *   dq         [B, T, Hq, d] fp32, overwritten
 *   dk, dv     [B, Lcap, Hkv, d] fp32, overwritten: keys no query reads get 0
 *   ws         >= infllmv2_backward_workspace_size(params, B, T, max_ctx, Hq, Hkv, d) bytes, 256-byte aligned
 * dk / dv are sums of fp32 atomics: equal up to rounding order between runs.
 */
size_t infllmv2_backward_workspace_size(const infllmv2_params* params, int batch, int max_q, int max_ctx, int hq,
                                        int hkv, int head_dim);
int infllmv2_sparse_attn_backward(const void* q, int batch, int num_q, int hq, int hkv, int head_dim, const void* k,
                                  const void* v, int lcap, const int32_t* q_ctx, const int32_t* ctx_lens, int max_ctx,
                                  const int32_t* idx, const int32_t* cnt, const infllmv2_params* params,
                                  const void* out, const float* lse, const void* dout, float* dq, float* dk,
                                  float* dv, void* ws, size_t ws_bytes, infllmv2_stream_t stream);

/*
 * The draft model's sliding-window attention (MiniCPM4 technical details, section "speculative sampling,
 * quantisation and long text", long-context bullet: the draft model attends with a sliding window; the
 * pages give no window size).  One query per sequence attends to its last `window` keys:
 *   out[b, h, :] = sum_{i in [max(0, n - window), n)} softmax_i(scale * q . k_i) v_i,  n = ctx_lens[b]
 * Same layouts, scale rule and workspace as infllmv2_dense_attn_decode (size it with the same call and
 * max_ctx; the window needs at most that much).  window >= 1, else INFLLMV2_ERR_INVALID_ARG.
 */
int infllmv2_window_attn_decode(const void* q, int batch, int hq, int hkv, int head_dim, const void* k, const void* v,
                                int lcap, const int32_t* ctx_lens, int max_ctx, int window, float softmax_scale,
                                void* out, float* lse, void* ws, size_t ws_bytes, infllmv2_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* INFLLMV2_H */

// internal.h -- launchers shared between the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "../../include/infllmv2.h"

namespace iv2 {

// Raise a kernel's dynamic shared-memory limit once per (kernel, device), so that stream captures after
// the first call see no attribute calls.  Returns the CUDA error of the attribute call.
cudaError_t ensure_smem_impl(const void* func, size_t bytes);
template <typename F>
inline cudaError_t ensure_smem(F* func, size_t bytes)
{
    return ensure_smem_impl(reinterpret_cast<const void*>(func), bytes);
}

// Launch with programmatic stream serialization: the kernel may be scheduled while the previous kernel of
// the stream is still running; it waits for it with griddepcontrol.wait (pdl_wait) before any global access.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The same with a thread-block cluster of `cluster_x` CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, int cluster_x, size_t smem,
                                      cudaStream_t s, Args&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// 3-D bf16 TMA map with 128-byte swizzle over rows of `inner` elements: dims {inner, mid, outer}, box
// {64, box_mid, box_outer}; false when the driver entry point is missing or the encoder rejects the shape
bool make_tma_map_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                       uint64_t mid_stride_bytes, uint64_t outer_stride_bytes, uint32_t box_mid, uint32_t box_outer);

// Resolved per-call description of a set of query rows.
struct QueryRows {
    const void* q;            // [B, T, Hq, d] bf16, or packed [cu_q[B], Hq, d] when cu_q is set
    int B, T, Hq, Hkv, D;     // packed: T = the longest sequence's query count
    const int32_t* q_ctx;     // [B*T] or null
    const int32_t* ctx_lens;  // [B] (used when q_ctx is null)
    int same_ctx;             // q_ctx null: 1 -> every query of b sees ctx_lens[b] keys (tree drafts),
                              //             0 -> causal tail, n = ctx_lens[b] - T_b + t + 1
    int max_ctx;
    const int32_t* cu_q = nullptr;  // packed variable-length batch: sequence b's queries are rows
                                    // [cu_q[b], cu_q[b + 1]) (device, B + 1 entries); null: b * T + t
    const int32_t* cu_k = nullptr;  // with cu_q: sequence b has L_b = cu_k[b + 1] - cu_k[b] keys (device)
    long q_rows = 0;                // rows of q (host; B * T, or cu_q[B] when packed)
};

// number of queries of sequence b, and the row of query (b, t) in q / out / lse (idx / cnt: row * Hkv + g)
__host__ __device__ inline int q_len(const QueryRows& qr, int b)
{
    return qr.cu_q ? qr.cu_q[b + 1] - qr.cu_q[b] : qr.T;
}
__host__ __device__ inline long q_row(const QueryRows& qr, int b, int t)
{
    return qr.cu_q ? (long)qr.cu_q[b] + t : (long)b * qr.T + t;
}

// context length n of query (b, t)
__host__ __device__ inline int query_ctx(const QueryRows& qr, int b, int t)
{
    if (qr.q_ctx) return qr.q_ctx[b * qr.T + t];
    if (qr.cu_q) return (qr.cu_k[b + 1] - qr.cu_k[b]) - q_len(qr, b) + t + 1;  // the last T_b of L_b keys
    return qr.same_ctx ? qr.ctx_lens[b] : qr.ctx_lens[b] - q_len(qr, b) + t + 1;
}

// Where sequence b's keys and values live, as rows of [rows, Hkv, d] bf16 arrays:
//   contiguous (cu and table null): position i is row b * Lcap + i;
//   packed (cu set):                row cu[b] + i, sequences back to back (cu: device, B + 1 entries);
//   paged (table set):              row table[b * max_pages + i / 64] * 64 + i % 64 of a pool of num_pages
//                                   pages of 64 positions: one page holds one context block.
// A page id outside [0, num_pages) is never dereferenced: its positions read as zeros and are not written.
struct KvRows {
    int Lcap = 0;
    const int32_t* cu = nullptr;
    const int32_t* table = nullptr;
    int max_pages = 0, num_pages = 0;
    long rows = 0;  // rows the arrays hold (host): B * Lcap, cu[B], or num_pages * 64
};

// first row of context block blk of sequence b, or -1 when a paged cache maps it to no page
__device__ __forceinline__ long kv_block_row(const KvRows& kr, int b, int blk)
{
    if (kr.table) {
        if (blk < 0 || blk >= kr.max_pages) return -1;
        const int page = __ldg(kr.table + (size_t)b * kr.max_pages + blk);
        return (page >= 0 && page < kr.num_pages) ? (long)page * 64 : -1;
    }
    return (kr.cu ? (long)kr.cu[b] : (long)b * kr.Lcap) + (long)blk * 64;
}

// the row of position i of sequence b (-1: unmapped page)
__device__ __forceinline__ long kv_pos_row(const KvRows& kr, int b, int i)
{
    const long r0 = kv_block_row(kr, b, i >> 6);
    return r0 < 0 ? -1 : r0 + (i & 63);
}

inline KvRows kv_contiguous(int B, int Lcap)
{
    KvRows kr;
    kr.Lcap = Lcap;
    kr.rows = (long)B * Lcap;
    return kr;
}

struct MethodConsts {
    int topk, init_blocks, local_blocks, dense_len, membership;
    float scale;              // softmax scale (natural units)
    int kmax;                 // topk + init + local
    int window;               // > 0: attend to the last `window` keys only (sliding window); 0: off
    int lse_stride;           // <= 1: exact LSE; s > 1: LSE estimated from every s-th visible kernel
};

// rows (sequence x query x KV group) one split-attention launch handles
constexpr int kMaxSplitRows = 1 << 16;

// Argument checks of the two-call decode attention (api.cu): the status the workspace entry point would
// return before its workspace check, the method constants, and the number of KV splits per row.  Shared with
// the allocation-free entry point, so that both refuse exactly the same calls.
int check_decode_attn(const void* q, int batch, int hq, int hkv, int head_dim, const void* k, const void* v, int lcap,
                      const int32_t* ctx_lens, int max_ctx, const int32_t* idx, const int32_t* cnt,
                      const infllmv2_params* params, const void* out, const float* lse, MethodConsts* mc,
                      int* nsplit);

// scoring path: true -> split-kernel scan + per-row select (needs workspace), false -> token tiles
bool score_uses_scan_path(int B, int T, int G, int D, int max_ctx);
// workspace bytes of the scan path / of the split attention (256-byte multiples)
size_t score_ws_bytes(int rows, int max_ctx);
size_t attn_ws_bytes(int rows, int nsplit);
// CTAs per row of the split attention for a block list of max_blocks entries
int attn_split_count(int max_blocks);
// largest block list the split attention handles for these sizes
int attn_split_max_blocks(int max_ctx, int kmax, int dense_len, bool dense_all, int window = 0);

// old_lens null: every sequence starts from 0 keys; new_lens null (packed keys only): L_b = cu[b + 1] - cu[b]
cudaError_t launch_kernel_pool(const void* k, int B, const KvRows& kr, int Hkv, int D, const int32_t* old_lens,
                               const int32_t* new_lens, int max_new_keys, void* kern, int nk_cap, cudaStream_t s);

cudaError_t launch_kernel_pool_backward(const float* dkern, int B, int Lcap, int Hkv, int D, const int32_t* lens,
                                        int max_len, int nk_cap, float* dk, bool accumulate, cudaStream_t s);

cudaError_t launch_kv_append(const void* k_new, const void* v_new, int B, int Hkv, int D, const int32_t* pos,
                             void* k_cache, void* v_cache, const KvRows& kr, cudaStream_t s);

cudaError_t launch_score_topk(const QueryRows& qr, const void* kern, int nk_cap, const MethodConsts& mc,
                              int32_t* idx, int32_t* cnt, void* ws, cudaStream_t s);

// the token-tile scoring on tcgen05/TMEM (16 heads per group, d = 128, at most 2048 context blocks);
// cudaErrorNotSupported otherwise
bool score_tc_supported(const QueryRows& qr, int nb_max);
cudaError_t launch_score_tc(const QueryRows& qr, const void* kern, int nk_cap, const MethodConsts& mc, int nb_max,
                            int32_t* idx, int32_t* cnt, cudaStream_t s);
int score_tc_error_flag_read_and_clear();

// attention over selected blocks (or all blocks when dense_all); prefill style: one warp per query row
cudaError_t launch_attn_rows(const QueryRows& qr, const void* k, const void* v, const KvRows& kr, const int32_t* idx,
                             const int32_t* cnt, const MethodConsts& mc, bool dense_all, void* out, float* lse,
                             cudaStream_t s);

// the same on tcgen05/TMEM with TMA-staged K/V (16 heads per group, d = 128); cudaErrorNotSupported otherwise
bool attn_tc_supported(const QueryRows& qr);
cudaError_t launch_attn_rows_tc(const QueryRows& qr, const void* k, const void* v, const KvRows& kr, const int32_t* idx,
                                const int32_t* cnt, const MethodConsts& mc, bool dense_all, void* out, float* lse,
                                cudaStream_t s);
// device-side error flag of the bounded waits (1 = a wait ran out); reading clears it; -1 on a CUDA error
int tc_error_flag_read_and_clear();

// one decode step (scoring, top-k, sparse attention) in a single cluster kernel; cudaErrorNotSupported when
// the shape is outside what it handles
bool decode_fused_supported(const QueryRows& qr, const MethodConsts& mc);
// pool_new: first pool, into kern, the kernel completed by each row's last key (kernel_pool of old = n - 1,
// new = n, done by the CTA that owns it)
cudaError_t launch_decode_fused(const QueryRows& qr, const void* kern, int nk_cap, const MethodConsts& mc,
                                const void* k, const void* v, const KvRows& kr, int32_t* idx, int32_t* cnt, void* out,
                                float* lse, cudaStream_t s, bool pool_new = false);
int fused_error_flag_read_and_clear();
int fused_set_first_wait_limit(unsigned polls);  // testing only
unsigned test_first_wait_limit();                // the value set (0: the normal waits)

// attention split over the selected blocks across CTAs, merged by LSE (decode and tree verification)
cudaError_t launch_attn_split(const QueryRows& qr, const void* k, const void* v, const KvRows& kr, const int32_t* idx,
                              const int32_t* cnt, const MethodConsts& mc, bool dense_all, const void* k_draft,
                              const void* v_draft, const uint32_t* tree_mask, void* out, float* lse, void* ws,
                              cudaStream_t s);

// gradients of the attention for a fixed selection (prefill layout): workspace bytes, and the launches
size_t attn_bwd_ws_bytes(int B, int T, int Hq, int Hkv, int max_ctx, int kmax, int dense_len, bool dense_all);
cudaError_t launch_attn_backward(const QueryRows& qr, const void* k, const void* v, int Lcap, const int32_t* idx,
                                 const int32_t* cnt, const MethodConsts& mc, bool dense_all, const void* out,
                                 const float* lse, const void* dout, float* dq, float* dk, float* dv, void* ws,
                                 cudaStream_t s);

// dq of the backward on tcgen05/TMEM (16 heads per group, d = 128); cudaErrorNotSupported otherwise
bool bwd_dq_tc_supported(const QueryRows& qr);
cudaError_t launch_bwd_dq_tc(const QueryRows& qr, const void* k, const void* v, int Lcap, const int32_t* idx,
                             const int32_t* cnt, const MethodConsts& mc, bool dense_all, const float* lse,
                             const float* dsum, const void* dout, float* dq, cudaStream_t s);
bool bwd_dkdv_tc_supported(const QueryRows& qr);
cudaError_t launch_bwd_dkdv_tc(const QueryRows& qr, const void* k, const void* v, int Lcap, const MethodConsts& mc,
                               int nb, const float* lse, const float* dsum, const void* dout, const int* counts,
                               const int* offsets, const int* tokens, const int* nitems, const int* item_list,
                               const int* item_start, int cap, int max_items, float* dk, float* dv, cudaStream_t s);
int bwd_tc_error_flag_read_and_clear();

}  // namespace iv2

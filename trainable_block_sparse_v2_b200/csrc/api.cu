// api.cu -- the C ABI of libinfllmv2.so (declared in include/infllmv2.h).
//
// Every entry point validates its arguments on the host and returns a status before launching anything
// when they are wrong; then it enqueues the kernels on the caller's stream.  The library allocates no
// memory and keeps no state between calls.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/infllmv2.h"
#include "common.cuh"
#include "internal.h"

namespace iv2 {

cudaError_t ensure_smem_impl(const void* func, size_t bytes)
{
    struct Entry {
        const void* func;
        int dev;
        size_t bytes;
    };
    static Entry table[256];
    static int n = 0;
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
        if (table[i].func == func && table[i].dev == dev && table[i].bytes >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && n < 256) table[n++] = Entry{func, dev, bytes};
    return e;
}

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// the driver's tensor-map encoder, looked up once through the runtime (no link-time libcuda dependency)
EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

}  // namespace

bool make_tma_map_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                       uint64_t mid_stride_bytes, uint64_t outer_stride_bytes, uint32_t box_mid, uint32_t box_outer)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)inner, mid, outer};
    const cuuint64_t strides[2] = {mid_stride_bytes, outer_stride_bytes};
    const cuuint32_t box[3] = {64, box_mid, box_outer};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace iv2

using iv2::MethodConsts;
using iv2::QueryRows;

namespace {

constexpr int kVersion = 100;  // 0.1.0

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int nk_of(long n) { return n >= iv2::kKernelSize ? (int)((n - iv2::kKernelSize) / iv2::kKernelStride + 1) : 0; }

constexpr int kMaxBlocks = 4096;  // contexts up to 256K keys

int check_params(const infllmv2_params* p)
{
    if (!p) return INFLLMV2_ERR_INVALID_ARG;
    if (p->topk < 0 || p->init_blocks < 0 || p->local_blocks < 0 || p->dense_len < 0) return INFLLMV2_ERR_INVALID_ARG;
    // far past any supported context (kMaxBlocks), and small enough that their sum stays an int
    constexpr int kMaxCount = 1 << 24;
    if (p->topk > kMaxCount || p->init_blocks > kMaxCount || p->local_blocks > kMaxCount)
        return INFLLMV2_ERR_INVALID_ARG;
    if (p->membership != 0 && p->membership != 1) return INFLLMV2_ERR_INVALID_ARG;
    if (p->topk + p->init_blocks + p->local_blocks < 1) return INFLLMV2_ERR_INVALID_ARG;
    if (!(p->softmax_scale == p->softmax_scale) || std::isinf(p->softmax_scale)) return INFLLMV2_ERR_INVALID_ARG;
    if (p->block_size != iv2::kBlock || p->kernel_size != iv2::kKernelSize || p->kernel_stride != iv2::kKernelStride)
        return INFLLMV2_ERR_UNSUPPORTED;
    if (p->lse_stride < 0) return INFLLMV2_ERR_INVALID_ARG;
    if (p->lse_stride > 1 && p->lse_stride != 2 && p->lse_stride != 4 && p->lse_stride != 8)
        return INFLLMV2_ERR_UNSUPPORTED;
    return INFLLMV2_OK;
}

MethodConsts consts_of(const infllmv2_params* p, int d)
{
    MethodConsts mc{};
    mc.topk = p->topk;
    mc.init_blocks = p->init_blocks;
    mc.local_blocks = p->local_blocks;
    mc.dense_len = p->dense_len;
    mc.membership = p->membership;
    mc.scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt((float)d);
    mc.kmax = p->topk + p->init_blocks + p->local_blocks;
    mc.window = 0;
    mc.lse_stride = p->lse_stride > 1 ? p->lse_stride : 1;
    return mc;
}

MethodConsts dense_consts(float scale, int d)
{
    MethodConsts mc{};
    mc.topk = 0;
    mc.init_blocks = 0;
    mc.local_blocks = 0;
    mc.dense_len = 0;
    mc.membership = 0;
    mc.scale = scale > 0.f ? scale : 1.0f / std::sqrt((float)d);
    mc.kmax = 1;
    return mc;
}

int check_heads(int batch, int nq, int hq, int hkv, int d)
{
    if (batch < 1 || nq < 1 || hq < 1 || hkv < 1) return INFLLMV2_ERR_INVALID_ARG;
    if (hq % hkv != 0) return INFLLMV2_ERR_INVALID_ARG;
    const int G = hq / hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return INFLLMV2_ERR_UNSUPPORTED;
    if (d != 64 && d != 128) return INFLLMV2_ERR_UNSUPPORTED;
    if ((long)batch * nq * hkv > (1L << 30)) return INFLLMV2_ERR_UNSUPPORTED;
    return INFLLMV2_OK;
}

int check_ptr16(const void* p) { return (p && aligned(p, 16)) ? INFLLMV2_OK : INFLLMV2_ERR_INVALID_ARG; }
int check_ptr4(const void* p) { return (p && aligned(p, 4)) ? INFLLMV2_OK : INFLLMV2_ERR_INVALID_ARG; }
int check_opt4(const void* p) { return (!p || aligned(p, 4)) ? INFLLMV2_OK : INFLLMV2_ERR_INVALID_ARG; }

int check_ctx(int max_ctx, int lcap)
{
    if (max_ctx < 1) return INFLLMV2_ERR_INVALID_ARG;
    if (lcap >= 0 && max_ctx > lcap) return INFLLMV2_ERR_INVALID_ARG;
    if ((max_ctx - 1) / iv2::kBlock + 1 > kMaxBlocks) return INFLLMV2_ERR_UNSUPPORTED;
    return INFLLMV2_OK;
}

int check_ws(void* ws, size_t ws_bytes, size_t need)
{
    if (need == 0) return INFLLMV2_OK;
    if (!ws || !aligned(ws, 256) || ws_bytes < need) return INFLLMV2_ERR_WORKSPACE;
    return INFLLMV2_OK;
}

int launched(cudaError_t e) { return e == cudaSuccess ? INFLLMV2_OK : INFLLMV2_ERR_CUDA; }

#define IV2_TRY(expr)                        \
    do {                                     \
        const int _st = (expr);              \
        if (_st != INFLLMV2_OK) return _st;  \
    } while (0)

size_t score_need(int batch, int nq, int hq, int hkv, int d, int max_ctx)
{
    if (!iv2::score_uses_scan_path(batch, nq, hq / hkv, d, max_ctx)) return 0;
    return iv2::score_ws_bytes(batch * nq * hkv, max_ctx);
}

size_t split_need(int rows, int max_ctx, int kmax, int dense_len, bool dense_all, bool draft, int window = 0)
{
    const int nsplit =
        iv2::attn_split_count(iv2::attn_split_max_blocks(max_ctx, kmax, dense_len, dense_all, window)) +
        (draft ? 1 : 0);
    return iv2::attn_ws_bytes(rows, nsplit);
}

QueryRows rows_of(const void* q, int B, int T, int hq, int hkv, int d, const int32_t* q_ctx, const int32_t* ctx_lens,
                  int same_ctx, int max_ctx)
{
    QueryRows qr;
    qr.q = q;
    qr.B = B;
    qr.T = T;
    qr.Hq = hq;
    qr.Hkv = hkv;
    qr.D = d;
    qr.q_ctx = q_ctx;
    qr.ctx_lens = ctx_lens;
    qr.same_ctx = same_ctx;
    qr.max_ctx = max_ctx;
    qr.cu_q = nullptr;
    qr.q_rows = (long)B * T;
    return qr;
}

}  // namespace

// Argument checks and method constants of the two-call decode attention, shared by
// infllmv2_sparse_attn_decode and infllmv2_sparse_attn_decode_noalloc so that both refuse the same calls.
int iv2::check_decode_attn(const void* q, int batch, int hq, int hkv, int head_dim, const void* k, const void* v,
                           int lcap, const int32_t* ctx_lens, int max_ctx, const int32_t* idx, const int32_t* cnt,
                           const infllmv2_params* params, const void* out, const float* lse, MethodConsts* mc,
                           int* nsplit)
{
    IV2_TRY(check_params(params));
    IV2_TRY(check_heads(batch, 1, hq, hkv, head_dim));
    IV2_TRY(check_ptr16(q));
    IV2_TRY(check_ptr16(k));
    IV2_TRY(check_ptr16(v));
    IV2_TRY(check_ptr16(out));
    IV2_TRY(check_ptr4(idx));
    IV2_TRY(check_ptr4(cnt));
    IV2_TRY(check_ptr4(ctx_lens));
    IV2_TRY(check_opt4(lse));
    IV2_TRY(check_ctx(max_ctx, lcap));
    *mc = consts_of(params, head_dim);
    if (batch * hkv > iv2::kMaxSplitRows) return INFLLMV2_ERR_UNSUPPORTED;
    *nsplit = iv2::attn_split_count(iv2::attn_split_max_blocks(max_ctx, mc->kmax, mc->dense_len, false));
    return INFLLMV2_OK;
}

// ---- packed variable-length batches and paged caches ----
namespace {

constexpr int kMaxPagesInPool = 1 << 24;  // page * 64 rows stays an int

int check_pages(const void* pool0, const void* pool1, int num_pages, const int32_t* table, int max_pages)
{
    IV2_TRY(check_ptr16(pool0));
    if (pool1) IV2_TRY(check_ptr16(pool1));
    IV2_TRY(check_ptr4(table));
    if (num_pages < 1 || max_pages < 1) return INFLLMV2_ERR_INVALID_ARG;
    if (num_pages > kMaxPagesInPool || max_pages > kMaxBlocks) return INFLLMV2_ERR_UNSUPPORTED;
    return INFLLMV2_OK;
}

iv2::KvRows kv_paged(const int32_t* table, int max_pages, int num_pages)
{
    iv2::KvRows kr;
    kr.Lcap = max_pages * iv2::kBlock;  // positions the table can address
    kr.table = table;
    kr.max_pages = max_pages;
    kr.num_pages = num_pages;
    kr.rows = (long)num_pages * iv2::kBlock;
    return kr;
}

iv2::KvRows kv_packed(const int32_t* cu, long total)
{
    iv2::KvRows kr;
    kr.cu = cu;
    kr.rows = total;
    return kr;
}

}  // namespace

extern "C" {

const char* infllmv2_status_string(int status)
{
    switch (status) {
    case INFLLMV2_OK: return "ok";
    case INFLLMV2_ERR_INVALID_ARG: return "invalid argument";
    case INFLLMV2_ERR_UNSUPPORTED: return "unsupported configuration";
    case INFLLMV2_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case INFLLMV2_ERR_CUDA: return "CUDA launch failed";
    case INFLLMV2_ERR_TIMEOUT: return "timeout";
    default: return "unknown status";
    }
}

int infllmv2_version(void) { return kVersion; }

int infllmv2_device_status(void)
{
    const int f = iv2::tc_error_flag_read_and_clear();
    const int h = iv2::fused_error_flag_read_and_clear();
    const int sc = iv2::score_tc_error_flag_read_and_clear();
    const int bw = iv2::bwd_tc_error_flag_read_and_clear();
    if (f < 0 || h < 0 || sc < 0 || bw < 0) return INFLLMV2_ERR_CUDA;
    return (f || h || sc || bw) ? INFLLMV2_ERR_TIMEOUT : INFLLMV2_OK;
}

size_t infllmv2_workspace_size(const infllmv2_params* params, int batch, int max_q, int max_ctx, int hq, int hkv,
                               int head_dim)
{
    if (check_params(params) != INFLLMV2_OK) return 0;
    if (check_heads(batch, max_q, hq, hkv, head_dim) != INFLLMV2_OK) return 0;
    if (check_ctx(max_ctx, -1) != INFLLMV2_OK) return 0;
    const int kmax = params->topk + params->init_blocks + params->local_blocks;
    size_t need = score_need(batch, max_q, hq, hkv, head_dim, max_ctx);
    const int rows = batch * max_q * hkv;
    const size_t attn = split_need(rows, max_ctx, kmax, params->dense_len, true, true);
    if (attn > need) need = attn;
    return need < 256 ? 256 : need;
}

int infllmv2_kernel_pool(const void* k, int batch, int lcap, int hkv, int head_dim, const int32_t* old_lens,
                         const int32_t* new_lens, int max_new_keys, const infllmv2_params* params, void* kern,
                         int nk_cap, infllmv2_stream_t stream)
{
    IV2_TRY(check_params(params));
    IV2_TRY(check_heads(batch, 1, hkv, hkv, head_dim));
    IV2_TRY(check_ptr16(k));
    IV2_TRY(check_ptr16(kern));
    IV2_TRY(check_ptr4(old_lens));
    IV2_TRY(check_ptr4(new_lens));
    if (lcap < 1 || max_new_keys < 0 || nk_cap < 1 || max_new_keys > lcap) return INFLLMV2_ERR_INVALID_ARG;
    if (nk_cap < nk_of(max_new_keys)) return INFLLMV2_ERR_INVALID_ARG;
    if (max_new_keys == 0) return INFLLMV2_OK;
    return launched(iv2::launch_kernel_pool(k, batch, iv2::kv_contiguous(batch, lcap), hkv, head_dim, old_lens, new_lens,
                                            max_new_keys, kern, nk_cap, (cudaStream_t)stream));
}

int infllmv2_kernel_pool_backward(const float* dkern, int batch, int lcap, int hkv, int head_dim, const int32_t* lens,
                                  int max_len, const infllmv2_params* params, int nk_cap, float* dk, int accumulate,
                                  infllmv2_stream_t stream)
{
    IV2_TRY(check_params(params));
    IV2_TRY(check_heads(batch, 1, hkv, hkv, head_dim));
    IV2_TRY(check_ptr16(dkern));
    IV2_TRY(check_ptr16(dk));
    IV2_TRY(check_ptr4(lens));
    if (lcap < 1 || max_len < 0 || max_len > lcap || nk_cap < 1 || (accumulate != 0 && accumulate != 1))
        return INFLLMV2_ERR_INVALID_ARG;
    if (nk_cap < nk_of(max_len)) return INFLLMV2_ERR_INVALID_ARG;
    if ((long)batch * hkv > 65535) return INFLLMV2_ERR_UNSUPPORTED;
    if (max_len == 0) return INFLLMV2_OK;
    return launched(iv2::launch_kernel_pool_backward(dkern, batch, lcap, hkv, head_dim, lens, max_len, nk_cap, dk,
                                                     accumulate != 0, (cudaStream_t)stream));
}

int infllmv2_kv_append(const void* k_new, const void* v_new, int batch, int hkv, int head_dim, const int32_t* pos,
                       void* k_cache, void* v_cache, int lcap, infllmv2_stream_t stream)
{
    IV2_TRY(check_heads(batch, 1, hkv, hkv, head_dim));
    IV2_TRY(check_ptr16(k_new));
    IV2_TRY(check_ptr16(v_new));
    IV2_TRY(check_ptr16(k_cache));
    IV2_TRY(check_ptr16(v_cache));
    IV2_TRY(check_ptr4(pos));
    if (lcap < 1) return INFLLMV2_ERR_INVALID_ARG;
    return launched(iv2::launch_kv_append(k_new, v_new, batch, hkv, head_dim, pos, k_cache, v_cache,
                                          iv2::kv_contiguous(batch, lcap), (cudaStream_t)stream));
}

int infllmv2_block_score_topk(const void* q, int batch, int num_q, int hq, int hkv, int head_dim,
                              const int32_t* q_ctx, const int32_t* ctx_lens, int max_ctx, const void* kern,
                              int nk_cap, const infllmv2_params* params, int32_t* idx, int32_t* cnt, void* ws,
                              size_t ws_bytes, infllmv2_stream_t stream)
{
    IV2_TRY(check_params(params));
    IV2_TRY(check_heads(batch, num_q, hq, hkv, head_dim));
    IV2_TRY(check_ptr16(q));
    IV2_TRY(check_ptr16(kern));
    IV2_TRY(check_ptr4(idx));
    IV2_TRY(check_ptr4(cnt));
    IV2_TRY(check_opt4(q_ctx));
    IV2_TRY(check_opt4(ctx_lens));
    if (!q_ctx && !ctx_lens) return INFLLMV2_ERR_INVALID_ARG;
    IV2_TRY(check_ctx(max_ctx, -1));
    if (nk_cap < 1 || nk_cap < nk_of(max_ctx)) return INFLLMV2_ERR_INVALID_ARG;
    IV2_TRY(check_ws(ws, ws_bytes, score_need(batch, num_q, hq, hkv, head_dim, max_ctx)));
    const QueryRows qr = rows_of(q, batch, num_q, hq, hkv, head_dim, q_ctx, ctx_lens, 0, max_ctx);
    // the LSE estimate exists on the tensor-core prefill scoring only
    if (params->lse_stride > 1 && (iv2::score_uses_scan_path(batch, num_q, hq / hkv, head_dim, max_ctx) ||
                                   !iv2::score_tc_supported(qr, (max_ctx - 1) / iv2::kBlock + 1)))
        return INFLLMV2_ERR_UNSUPPORTED;
    return launched(iv2::launch_score_topk(qr, kern, nk_cap, consts_of(params, head_dim), idx, cnt, ws,
                                           (cudaStream_t)stream));
}

int infllmv2_sparse_attn_prefill(const void* q, int batch, int num_q, int hq, int hkv, int head_dim, const void* k,
                                 const void* v, int lcap, const int32_t* q_ctx, const int32_t* ctx_lens, int max_ctx,
                                 const int32_t* idx, const int32_t* cnt, const infllmv2_params* params, void* out,
                                 float* lse, void* ws, size_t ws_bytes, infllmv2_stream_t stream)
{
    (void)ws;
    (void)ws_bytes;
    IV2_TRY(check_params(params));
    IV2_TRY(check_heads(batch, num_q, hq, hkv, head_dim));
    IV2_TRY(check_ptr16(q));
    IV2_TRY(check_ptr16(k));
    IV2_TRY(check_ptr16(v));
    IV2_TRY(check_ptr16(out));
    IV2_TRY(check_ptr4(idx));
    IV2_TRY(check_ptr4(cnt));
    IV2_TRY(check_opt4(lse));
    IV2_TRY(check_opt4(q_ctx));
    IV2_TRY(check_opt4(ctx_lens));
    if (!q_ctx && !ctx_lens) return INFLLMV2_ERR_INVALID_ARG;
    IV2_TRY(check_ctx(max_ctx, lcap));
    const QueryRows qr = rows_of(q, batch, num_q, hq, hkv, head_dim, q_ctx, ctx_lens, 0, max_ctx);
    const MethodConsts mc = consts_of(params, head_dim);
    if (iv2::attn_tc_supported(qr)) {
        const cudaError_t e = iv2::launch_attn_rows_tc(qr, k, v, iv2::kv_contiguous(batch, lcap), idx, cnt, mc, false, out, lse,
                                                       (cudaStream_t)stream);
        if (e != cudaErrorNotSupported) return launched(e);
    }
    return launched(iv2::launch_attn_rows(qr, k, v, iv2::kv_contiguous(batch, lcap), idx, cnt, mc, false, out, lse, (cudaStream_t)stream));
}

int infllmv2_sparse_attn_decode(const void* q, int batch, int hq, int hkv, int head_dim, const void* k, const void* v,
                                int lcap, const int32_t* ctx_lens, int max_ctx, const int32_t* idx,
                                const int32_t* cnt, const infllmv2_params* params, void* out, float* lse, void* ws,
                                size_t ws_bytes, infllmv2_stream_t stream)
{
    MethodConsts mc;
    int nsplit = 0;
    IV2_TRY(iv2::check_decode_attn(q, batch, hq, hkv, head_dim, k, v, lcap, ctx_lens, max_ctx, idx, cnt, params, out,
                                   lse, &mc, &nsplit));
    IV2_TRY(check_ws(ws, ws_bytes, iv2::attn_ws_bytes(batch * hkv, nsplit)));
    const QueryRows qr = rows_of(q, batch, 1, hq, hkv, head_dim, nullptr, ctx_lens, 0, max_ctx);
    return launched(iv2::launch_attn_split(qr, k, v, iv2::kv_contiguous(batch, lcap), idx, cnt, mc, false, nullptr, nullptr, nullptr, out, lse,
                                           ws, (cudaStream_t)stream));
}

int infllmv2_sparse_decode_step(const void* q, int batch, int hq, int hkv, int head_dim, const void* kern, int nk_cap,
                                const void* k, const void* v, int lcap, const int32_t* ctx_lens, int max_ctx,
                                const infllmv2_params* params, int32_t* idx, int32_t* cnt, void* out, float* lse,
                                infllmv2_stream_t stream)
{
    IV2_TRY(check_params(params));
    if (params->lse_stride > 1) return INFLLMV2_ERR_UNSUPPORTED;  // the estimate is built for prefill scoring only
    IV2_TRY(check_heads(batch, 1, hq, hkv, head_dim));
    IV2_TRY(check_ptr16(q));
    IV2_TRY(check_ptr16(kern));
    IV2_TRY(check_ptr16(k));
    IV2_TRY(check_ptr16(v));
    IV2_TRY(check_ptr16(out));
    IV2_TRY(check_ptr4(ctx_lens));
    IV2_TRY(check_ptr4(idx));
    IV2_TRY(check_ptr4(cnt));
    IV2_TRY(check_opt4(lse));
    IV2_TRY(check_ctx(max_ctx, lcap));
    if (nk_cap < 1 || nk_cap < nk_of(max_ctx)) return INFLLMV2_ERR_INVALID_ARG;
    if (batch * hkv > 65535) return INFLLMV2_ERR_UNSUPPORTED;
    const MethodConsts mc = consts_of(params, head_dim);
    const QueryRows qr = rows_of(q, batch, 1, hq, hkv, head_dim, nullptr, ctx_lens, 0, max_ctx);
    if (!iv2::decode_fused_supported(qr, mc)) return INFLLMV2_ERR_UNSUPPORTED;
    return launched(iv2::launch_decode_fused(qr, kern, nk_cap, mc, k, v, iv2::kv_contiguous(batch, lcap), idx, cnt, out, lse,
                                             (cudaStream_t)stream));
}

int infllmv2_sparse_decode_step_pool(const void* q, int batch, int hq, int hkv, int head_dim, void* kern, int nk_cap,
                                const void* k, const void* v, int lcap, const int32_t* ctx_lens, int max_ctx,
                                const infllmv2_params* params, int32_t* idx, int32_t* cnt, void* out, float* lse,
                                infllmv2_stream_t stream)
{
    IV2_TRY(check_params(params));
    if (params->lse_stride > 1) return INFLLMV2_ERR_UNSUPPORTED;  // the estimate is built for prefill scoring only
    IV2_TRY(check_heads(batch, 1, hq, hkv, head_dim));
    IV2_TRY(check_ptr16(q));
    IV2_TRY(check_ptr16(kern));
    IV2_TRY(check_ptr16(k));
    IV2_TRY(check_ptr16(v));
    IV2_TRY(check_ptr16(out));
    IV2_TRY(check_ptr4(ctx_lens));
    IV2_TRY(check_ptr4(idx));
    IV2_TRY(check_ptr4(cnt));
    IV2_TRY(check_opt4(lse));
    IV2_TRY(check_ctx(max_ctx, lcap));
    if (nk_cap < 1 || nk_cap < nk_of(max_ctx)) return INFLLMV2_ERR_INVALID_ARG;
    if (batch * hkv > 65535) return INFLLMV2_ERR_UNSUPPORTED;
    const MethodConsts mc = consts_of(params, head_dim);
    const QueryRows qr = rows_of(q, batch, 1, hq, hkv, head_dim, nullptr, ctx_lens, 0, max_ctx);
    if (!iv2::decode_fused_supported(qr, mc)) return INFLLMV2_ERR_UNSUPPORTED;
    return launched(iv2::launch_decode_fused(qr, kern, nk_cap, mc, k, v, iv2::kv_contiguous(batch, lcap), idx, cnt, out, lse,
                                             (cudaStream_t)stream, true));
}

int infllmv2_sparse_attn_tree_verify(const void* q, int batch, int n_draft, int hq, int hkv, int head_dim,
                                     const void* k, const void* v, int lcap, const int32_t* prefix_lens, int max_ctx,
                                     const void* k_draft, const void* v_draft, const uint32_t* tree_mask,
                                     const int32_t* idx, const int32_t* cnt, const infllmv2_params* params, void* out,
                                     float* lse, void* ws, size_t ws_bytes, infllmv2_stream_t stream)
{
    IV2_TRY(check_params(params));
    IV2_TRY(check_heads(batch, n_draft, hq, hkv, head_dim));
    if (n_draft > 32) return INFLLMV2_ERR_UNSUPPORTED;
    IV2_TRY(check_ptr16(q));
    IV2_TRY(check_ptr16(k));
    IV2_TRY(check_ptr16(v));
    IV2_TRY(check_ptr16(k_draft));
    IV2_TRY(check_ptr16(v_draft));
    IV2_TRY(check_ptr16(out));
    IV2_TRY(check_ptr4(tree_mask));
    IV2_TRY(check_ptr4(idx));
    IV2_TRY(check_ptr4(cnt));
    IV2_TRY(check_ptr4(prefix_lens));
    IV2_TRY(check_opt4(lse));
    IV2_TRY(check_ctx(max_ctx, lcap));
    const MethodConsts mc = consts_of(params, head_dim);
    if (batch * n_draft * hkv > iv2::kMaxSplitRows) return INFLLMV2_ERR_UNSUPPORTED;
    IV2_TRY(check_ws(ws, ws_bytes, split_need(batch * n_draft * hkv, max_ctx, mc.kmax, mc.dense_len, false, true)));
    const QueryRows qr = rows_of(q, batch, n_draft, hq, hkv, head_dim, nullptr, prefix_lens, 1, max_ctx);
    return launched(iv2::launch_attn_split(qr, k, v, iv2::kv_contiguous(batch, lcap), idx, cnt, mc, false, k_draft, v_draft, tree_mask, out, lse,
                                           ws, (cudaStream_t)stream));
}

int infllmv2_dense_attn_prefill(const void* q, int batch, int num_q, int hq, int hkv, int head_dim, const void* k,
                                const void* v, int lcap, const int32_t* q_ctx, const int32_t* ctx_lens, int max_ctx,
                                float softmax_scale, void* out, float* lse, void* ws, size_t ws_bytes,
                                infllmv2_stream_t stream)
{
    (void)ws;
    (void)ws_bytes;
    IV2_TRY(check_heads(batch, num_q, hq, hkv, head_dim));
    if (!(softmax_scale == softmax_scale) || std::isinf(softmax_scale)) return INFLLMV2_ERR_INVALID_ARG;
    IV2_TRY(check_ptr16(q));
    IV2_TRY(check_ptr16(k));
    IV2_TRY(check_ptr16(v));
    IV2_TRY(check_ptr16(out));
    IV2_TRY(check_opt4(lse));
    IV2_TRY(check_opt4(q_ctx));
    IV2_TRY(check_opt4(ctx_lens));
    if (!q_ctx && !ctx_lens) return INFLLMV2_ERR_INVALID_ARG;
    IV2_TRY(check_ctx(max_ctx, lcap));
    const QueryRows qr = rows_of(q, batch, num_q, hq, hkv, head_dim, q_ctx, ctx_lens, 0, max_ctx);
    const MethodConsts mc = dense_consts(softmax_scale, head_dim);
    if (iv2::attn_tc_supported(qr)) {
        const cudaError_t e = iv2::launch_attn_rows_tc(qr, k, v, iv2::kv_contiguous(batch, lcap), nullptr, nullptr, mc, true, out, lse,
                                                       (cudaStream_t)stream);
        if (e != cudaErrorNotSupported) return launched(e);
    }
    return launched(iv2::launch_attn_rows(qr, k, v, iv2::kv_contiguous(batch, lcap), nullptr, nullptr, mc, true, out, lse, (cudaStream_t)stream));
}

size_t infllmv2_backward_workspace_size(const infllmv2_params* params, int batch, int max_q, int max_ctx, int hq,
                                        int hkv, int head_dim)
{
    if (check_params(params) != INFLLMV2_OK) return 0;
    if (check_heads(batch, max_q, hq, hkv, head_dim) != INFLLMV2_OK) return 0;
    if (check_ctx(max_ctx, -1) != INFLLMV2_OK) return 0;
    const int kmax = params->topk + params->init_blocks + params->local_blocks;
    // sized for the dense case too (idx == NULL), which bounds every sparse one
    const size_t sparse = iv2::attn_bwd_ws_bytes(batch, max_q, hq, hkv, max_ctx, kmax, params->dense_len, false);
    const size_t dense = iv2::attn_bwd_ws_bytes(batch, max_q, hq, hkv, max_ctx, kmax, params->dense_len, true);
    return sparse > dense ? sparse : dense;
}

int infllmv2_sparse_attn_backward(const void* q, int batch, int num_q, int hq, int hkv, int head_dim, const void* k,
                                  const void* v, int lcap, const int32_t* q_ctx, const int32_t* ctx_lens, int max_ctx,
                                  const int32_t* idx, const int32_t* cnt, const infllmv2_params* params,
                                  const void* out, const float* lse, const void* dout, float* dq, float* dk,
                                  float* dv, void* ws, size_t ws_bytes, infllmv2_stream_t stream)
{
    IV2_TRY(check_params(params));
    IV2_TRY(check_heads(batch, num_q, hq, hkv, head_dim));
    IV2_TRY(check_ptr16(q));
    IV2_TRY(check_ptr16(k));
    IV2_TRY(check_ptr16(v));
    IV2_TRY(check_ptr16(out));
    IV2_TRY(check_ptr16(dout));
    IV2_TRY(check_ptr16(dq));
    IV2_TRY(check_ptr16(dk));
    IV2_TRY(check_ptr16(dv));
    IV2_TRY(check_ptr4(lse));
    if ((idx == nullptr) != (cnt == nullptr)) return INFLLMV2_ERR_INVALID_ARG;
    IV2_TRY(check_opt4(idx));
    IV2_TRY(check_opt4(cnt));
    IV2_TRY(check_opt4(q_ctx));
    IV2_TRY(check_opt4(ctx_lens));
    if (!q_ctx && !ctx_lens) return INFLLMV2_ERR_INVALID_ARG;
    IV2_TRY(check_ctx(max_ctx, lcap));
    const bool dense_all = idx == nullptr;
    const MethodConsts mc = consts_of(params, head_dim);
    IV2_TRY(check_ws(ws, ws_bytes,
                     iv2::attn_bwd_ws_bytes(batch, num_q, hq, hkv, max_ctx, mc.kmax, mc.dense_len, dense_all)));
    const QueryRows qr = rows_of(q, batch, num_q, hq, hkv, head_dim, q_ctx, ctx_lens, 0, max_ctx);
    return launched(iv2::launch_attn_backward(qr, k, v, lcap, idx, cnt, mc, dense_all, out, lse, dout, dq, dk, dv, ws,
                                              (cudaStream_t)stream));
}

int infllmv2_dense_attn_decode(const void* q, int batch, int hq, int hkv, int head_dim, const void* k, const void* v,
                               int lcap, const int32_t* ctx_lens, int max_ctx, float softmax_scale, void* out,
                               float* lse, void* ws, size_t ws_bytes, infllmv2_stream_t stream)
{
    IV2_TRY(check_heads(batch, 1, hq, hkv, head_dim));
    if (!(softmax_scale == softmax_scale) || std::isinf(softmax_scale)) return INFLLMV2_ERR_INVALID_ARG;
    IV2_TRY(check_ptr16(q));
    IV2_TRY(check_ptr16(k));
    IV2_TRY(check_ptr16(v));
    IV2_TRY(check_ptr16(out));
    IV2_TRY(check_ptr4(ctx_lens));
    IV2_TRY(check_opt4(lse));
    IV2_TRY(check_ctx(max_ctx, lcap));
    const MethodConsts mc = dense_consts(softmax_scale, head_dim);
    if (batch * hkv > iv2::kMaxSplitRows) return INFLLMV2_ERR_UNSUPPORTED;
    IV2_TRY(check_ws(ws, ws_bytes, split_need(batch * hkv, max_ctx, mc.kmax, 0, true, false)));
    const QueryRows qr = rows_of(q, batch, 1, hq, hkv, head_dim, nullptr, ctx_lens, 0, max_ctx);
    return launched(iv2::launch_attn_split(qr, k, v, iv2::kv_contiguous(batch, lcap), nullptr, nullptr, mc, true, nullptr, nullptr, nullptr, out,
                                           lse, ws, (cudaStream_t)stream));
}

int infllmv2_window_attn_decode(const void* q, int batch, int hq, int hkv, int head_dim, const void* k, const void* v,
                                int lcap, const int32_t* ctx_lens, int max_ctx, int window, float softmax_scale,
                                void* out, float* lse, void* ws, size_t ws_bytes, infllmv2_stream_t stream)
{
    IV2_TRY(check_heads(batch, 1, hq, hkv, head_dim));
    if (!(softmax_scale == softmax_scale) || std::isinf(softmax_scale)) return INFLLMV2_ERR_INVALID_ARG;
    if (window < 1) return INFLLMV2_ERR_INVALID_ARG;
    IV2_TRY(check_ptr16(q));
    IV2_TRY(check_ptr16(k));
    IV2_TRY(check_ptr16(v));
    IV2_TRY(check_ptr16(out));
    IV2_TRY(check_ptr4(ctx_lens));
    IV2_TRY(check_opt4(lse));
    IV2_TRY(check_ctx(max_ctx, lcap));
    MethodConsts mc = dense_consts(softmax_scale, head_dim);
    mc.window = window;
    if (batch * hkv > iv2::kMaxSplitRows) return INFLLMV2_ERR_UNSUPPORTED;
    IV2_TRY(check_ws(ws, ws_bytes, split_need(batch * hkv, max_ctx, mc.kmax, 0, true, false, window)));
    const QueryRows qr = rows_of(q, batch, 1, hq, hkv, head_dim, nullptr, ctx_lens, 0, max_ctx);
    // one cluster launch (the decode step's kernel walking the window's blocks, partials merged on chip) when
    // the shape allows it; else the split attention and its merge
    if (batch * hkv <= 65535 && iv2::decode_fused_supported(qr, mc)) {
        const cudaError_t e = iv2::launch_decode_fused(qr, nullptr, 1, mc, k, v, iv2::kv_contiguous(batch, lcap), nullptr, nullptr, out, lse,
                                                       (cudaStream_t)stream);
        if (e != cudaErrorNotSupported) return launched(e);
    }
    return launched(iv2::launch_attn_split(qr, k, v, iv2::kv_contiguous(batch, lcap), nullptr, nullptr, mc, true, nullptr, nullptr, nullptr, out,
                                           lse, ws, (cudaStream_t)stream));
}


// ---- paged key/value cache ----
int infllmv2_kv_append_paged(const void* k_new, const void* v_new, int batch, int hkv, int head_dim, const int32_t* pos,
                             void* k_pages, void* v_pages, int num_pages, const int32_t* page_table, int max_pages,
                             infllmv2_stream_t stream)
{
    IV2_TRY(check_heads(batch, 1, hkv, hkv, head_dim));
    IV2_TRY(check_ptr16(k_new));
    IV2_TRY(check_ptr16(v_new));
    IV2_TRY(check_ptr4(pos));
    IV2_TRY(check_ptr16(v_pages));
    IV2_TRY(check_pages(k_pages, v_pages, num_pages, page_table, max_pages));
    return launched(iv2::launch_kv_append(k_new, v_new, batch, hkv, head_dim, pos, k_pages, v_pages,
                                          kv_paged(page_table, max_pages, num_pages), (cudaStream_t)stream));
}

int infllmv2_kernel_pool_paged(const void* k_pages, int num_pages, const int32_t* page_table, int max_pages,
                               int batch, int hkv, int head_dim, const int32_t* old_lens, const int32_t* new_lens,
                               int max_new_keys, const infllmv2_params* params, void* kern, int nk_cap,
                               infllmv2_stream_t stream)
{
    IV2_TRY(check_params(params));
    IV2_TRY(check_heads(batch, 1, hkv, hkv, head_dim));
    IV2_TRY(check_pages(k_pages, nullptr, num_pages, page_table, max_pages));
    IV2_TRY(check_ptr16(kern));
    IV2_TRY(check_ptr4(old_lens));
    IV2_TRY(check_ptr4(new_lens));
    const int lcap = max_pages * iv2::kBlock;
    if (max_new_keys < 0 || nk_cap < 1 || max_new_keys > lcap) return INFLLMV2_ERR_INVALID_ARG;
    if (nk_cap < nk_of(max_new_keys)) return INFLLMV2_ERR_INVALID_ARG;
    if (max_new_keys == 0) return INFLLMV2_OK;
    return launched(iv2::launch_kernel_pool(k_pages, batch, kv_paged(page_table, max_pages, num_pages), hkv, head_dim,
                                            old_lens, new_lens, max_new_keys, kern, nk_cap, (cudaStream_t)stream));
}

int infllmv2_sparse_decode_step_paged(const void* q, int batch, int hq, int hkv, int head_dim, const void* kern,
                                      int nk_cap, const void* k_pages, const void* v_pages, int num_pages,
                                      const int32_t* page_table, int max_pages, const int32_t* ctx_lens, int max_ctx,
                                      const infllmv2_params* params, int32_t* idx, int32_t* cnt, void* out,
                                      float* lse, infllmv2_stream_t stream)
{
    IV2_TRY(check_params(params));
    if (params->lse_stride > 1) return INFLLMV2_ERR_UNSUPPORTED;
    IV2_TRY(check_heads(batch, 1, hq, hkv, head_dim));
    IV2_TRY(check_ptr16(q));
    IV2_TRY(check_ptr16(kern));
    IV2_TRY(check_pages(k_pages, v_pages, num_pages, page_table, max_pages));
    IV2_TRY(check_ptr16(out));
    IV2_TRY(check_ptr4(ctx_lens));
    IV2_TRY(check_ptr4(idx));
    IV2_TRY(check_ptr4(cnt));
    IV2_TRY(check_opt4(lse));
    IV2_TRY(check_ctx(max_ctx, max_pages * iv2::kBlock));
    if (nk_cap < 1 || nk_cap < nk_of(max_ctx)) return INFLLMV2_ERR_INVALID_ARG;
    if (batch * hkv > 65535) return INFLLMV2_ERR_UNSUPPORTED;
    const MethodConsts mc = consts_of(params, head_dim);
    const QueryRows qr = rows_of(q, batch, 1, hq, hkv, head_dim, nullptr, ctx_lens, 0, max_ctx);
    if (!iv2::decode_fused_supported(qr, mc)) return INFLLMV2_ERR_UNSUPPORTED;
    return launched(iv2::launch_decode_fused(qr, kern, nk_cap, mc, k_pages, v_pages,
                                             kv_paged(page_table, max_pages, num_pages), idx, cnt, out, lse,
                                             (cudaStream_t)stream));
}

int infllmv2_sparse_attn_prefill_paged(const void* q, int batch, int num_q, int hq, int hkv, int head_dim,
                                       const void* k_pages, const void* v_pages, int num_pages,
                                       const int32_t* page_table, int max_pages, const int32_t* q_ctx,
                                       const int32_t* ctx_lens, int max_ctx, const int32_t* idx, const int32_t* cnt,
                                       const infllmv2_params* params, void* out, float* lse,
                                       infllmv2_stream_t stream)
{
    IV2_TRY(check_params(params));
    IV2_TRY(check_heads(batch, num_q, hq, hkv, head_dim));
    IV2_TRY(check_ptr16(q));
    IV2_TRY(check_pages(k_pages, v_pages, num_pages, page_table, max_pages));
    IV2_TRY(check_ptr16(out));
    IV2_TRY(check_ptr4(idx));
    IV2_TRY(check_ptr4(cnt));
    IV2_TRY(check_opt4(lse));
    IV2_TRY(check_opt4(q_ctx));
    IV2_TRY(check_opt4(ctx_lens));
    if (!q_ctx && !ctx_lens) return INFLLMV2_ERR_INVALID_ARG;
    IV2_TRY(check_ctx(max_ctx, max_pages * iv2::kBlock));
    const QueryRows qr = rows_of(q, batch, num_q, hq, hkv, head_dim, q_ctx, ctx_lens, 0, max_ctx);
    const MethodConsts mc = consts_of(params, head_dim);
    const iv2::KvRows kr = kv_paged(page_table, max_pages, num_pages);
    if (iv2::attn_tc_supported(qr)) {
        const cudaError_t e = iv2::launch_attn_rows_tc(qr, k_pages, v_pages, kr, idx, cnt, mc, false, out, lse,
                                                       (cudaStream_t)stream);
        if (e != cudaErrorNotSupported) return launched(e);
    }
    return launched(iv2::launch_attn_rows(qr, k_pages, v_pages, kr, idx, cnt, mc, false, out, lse, (cudaStream_t)stream));
}

// ---- packed variable-length prefill ----
int infllmv2_sparse_prefill_varlen(const void* q, const void* k, const void* v, int batch, int hq, int hkv, int head_dim,
                                   const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int total_q, int total_k,
                                   int max_seqlen_q, int max_seqlen_k, const infllmv2_params* params, void* kern,
                                   int nk_cap, int32_t* idx, int32_t* cnt, void* out, float* lse, void* ws,
                                   size_t ws_bytes, infllmv2_stream_t stream)
{
    IV2_TRY(check_params(params));
    IV2_TRY(check_heads(batch, max_seqlen_q < 1 ? 1 : max_seqlen_q, hq, hkv, head_dim));
    IV2_TRY(check_ptr16(q));
    IV2_TRY(check_ptr16(k));
    IV2_TRY(check_ptr16(v));
    IV2_TRY(check_ptr16(kern));
    IV2_TRY(check_ptr16(out));
    IV2_TRY(check_ptr4(idx));
    IV2_TRY(check_ptr4(cnt));
    IV2_TRY(check_ptr4(cu_seqlens_q));
    IV2_TRY(check_ptr4(cu_seqlens_k));
    IV2_TRY(check_opt4(lse));
    if (total_q < 0 || total_k < 0 || max_seqlen_q < 0 || max_seqlen_k < 0 || nk_cap < 1)
        return INFLLMV2_ERR_INVALID_ARG;
    if (max_seqlen_q > max_seqlen_k || max_seqlen_q > total_q || max_seqlen_k > total_k) return INFLLMV2_ERR_INVALID_ARG;
    if (max_seqlen_q == 0) return INFLLMV2_OK;  // no query anywhere
    IV2_TRY(check_ctx(max_seqlen_k, -1));
    if (nk_cap < nk_of(max_seqlen_k)) return INFLLMV2_ERR_INVALID_ARG;
    IV2_TRY(check_ws(ws, ws_bytes, score_need(batch, max_seqlen_q, hq, hkv, head_dim, max_seqlen_k)));
    if (params->lse_stride > 1 && (iv2::score_uses_scan_path(batch, max_seqlen_q, hq / hkv, head_dim, max_seqlen_k) ||
                                   head_dim != 128 || hq / hkv != 16))
        return INFLLMV2_ERR_UNSUPPORTED;
    QueryRows qr = rows_of(q, batch, max_seqlen_q, hq, hkv, head_dim, nullptr, nullptr, 0, max_seqlen_k);
    qr.cu_q = cu_seqlens_q;
    qr.cu_k = cu_seqlens_k;
    qr.q_rows = total_q;
    const MethodConsts mc = consts_of(params, head_dim);
    const iv2::KvRows kr = kv_packed(cu_seqlens_k, total_k);
    const cudaStream_t s = (cudaStream_t)stream;
    // 1. every complete kernel window of every sequence (old length 0, new length L_b)
    IV2_TRY(launched(iv2::launch_kernel_pool(k, batch, kr, hkv, head_dim, nullptr, nullptr, max_seqlen_k, kern, nk_cap,
                                             s)));
    // 2. scoring and top-k of every query
    IV2_TRY(launched(iv2::launch_score_topk(qr, kern, nk_cap, mc, idx, cnt, ws, s)));
    // 3. attention over the selected blocks
    if (iv2::attn_tc_supported(qr)) {
        const cudaError_t e = iv2::launch_attn_rows_tc(qr, k, v, kr, idx, cnt, mc, false, out, lse, s);
        if (e != cudaErrorNotSupported) return launched(e);
    }
    return launched(iv2::launch_attn_rows(qr, k, v, kr, idx, cnt, mc, false, out, lse, s));
}

int infllmv2_test_set_first_wait_limit(unsigned polls)
{
    return iv2::fused_set_first_wait_limit(polls) == 0 ? INFLLMV2_OK : INFLLMV2_ERR_CUDA;
}

}  // extern "C"

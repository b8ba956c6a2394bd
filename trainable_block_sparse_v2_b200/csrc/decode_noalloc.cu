// decode_noalloc.cu -- sparse decode attention whose scratch lives in a static device array.
//
// infllmv2_sparse_attn_decode needs a caller-provided workspace for the per-split partial results of its
// split-KV attention.  Some callers cannot provide one: code that may not call cudaMalloc after its
// start-up (a host process with a fixed memory budget handed out once, a plugin inside another runtime
// whose allocator it may not touch, a real-time loop that must never allocate).  This variant keeps those
// partials in one file-scope __device__ array instead, so the caller passes only inputs and outputs.
//
// The array is a fixed 4 MiB per GPU that loads the library, held until the process exits.  Its device
// address is looked up with cudaGetSymbolAddress once per device, on the first call made with that device
// current; make that first call before any stream capture.  Every call shares the array: calls whose
// kernels overlap on the GPU (other streams, other host threads) race on it.  The partials need no
// clearing: each call writes every partial it later reads.
#include <mutex>

#include "../../include/infllmv2.h"
#include "common.cuh"
#include "internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 4u << 20;  // 4 MiB

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// device address of the scratch array on the current device (looked up once per device)
cudaError_t scratch_address(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool aligned_to(const void* p, uintptr_t a) { return p && (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" int infllmv2_sparse_attn_decode_noalloc(const void* q, int batch, int hq, int hkv, int head_dim,
                                                   const void* k, const void* v, int lcap, const int32_t* ctx_lens,
                                                   int max_ctx, const int32_t* idx, const int32_t* cnt,
                                                   const infllmv2_params* params, void* out, float* lse,
                                                   infllmv2_stream_t stream)
{
    if (!params) return INFLLMV2_ERR_INVALID_ARG;
    if (params->block_size != iv2::kBlock || params->kernel_size != iv2::kKernelSize ||
        params->kernel_stride != iv2::kKernelStride)
        return INFLLMV2_ERR_UNSUPPORTED;
    if (params->topk < 0 || params->init_blocks < 0 || params->local_blocks < 0 || params->dense_len < 0 ||
        params->topk + params->init_blocks + params->local_blocks < 1 ||
        (params->membership != 0 && params->membership != 1) || !(params->softmax_scale == params->softmax_scale))
        return INFLLMV2_ERR_INVALID_ARG;
    if (batch < 1 || hq < 1 || hkv < 1 || hq % hkv != 0) return INFLLMV2_ERR_INVALID_ARG;
    const int G = hq / hkv;
    if ((G != 1 && G != 2 && G != 4 && G != 8 && G != 16) || (head_dim != 64 && head_dim != 128))
        return INFLLMV2_ERR_UNSUPPORTED;
    if (!aligned_to(q, 16) || !aligned_to(k, 16) || !aligned_to(v, 16) || !aligned_to(out, 16) ||
        !aligned_to(ctx_lens, 4) || !aligned_to(idx, 4) || !aligned_to(cnt, 4) || (lse && !aligned_to(lse, 4)))
        return INFLLMV2_ERR_INVALID_ARG;
    if (max_ctx < 1 || max_ctx > lcap) return INFLLMV2_ERR_INVALID_ARG;
    if ((max_ctx - 1) / iv2::kBlock + 1 > 4096) return INFLLMV2_ERR_UNSUPPORTED;

    iv2::MethodConsts mc{};
    mc.topk = params->topk;
    mc.init_blocks = params->init_blocks;
    mc.local_blocks = params->local_blocks;
    mc.dense_len = params->dense_len;
    mc.membership = params->membership;
    mc.scale = params->softmax_scale > 0.f ? params->softmax_scale : 1.0f / sqrtf((float)head_dim);
    mc.kmax = params->topk + params->init_blocks + params->local_blocks;
    // the partials of this call must fit the static array
    const int nsplit = iv2::attn_split_count(iv2::attn_split_max_blocks(max_ctx, mc.kmax, mc.dense_len, false));
    if (iv2::attn_ws_bytes(batch * hkv, nsplit) > kNoAllocScratchBytes) return INFLLMV2_ERR_WORKSPACE;

    void* scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return INFLLMV2_ERR_CUDA;

    iv2::QueryRows qr;
    qr.q = q;
    qr.B = batch;
    qr.T = 1;
    qr.Hq = hq;
    qr.Hkv = hkv;
    qr.D = head_dim;
    qr.q_ctx = nullptr;
    qr.ctx_lens = ctx_lens;
    qr.same_ctx = 0;
    qr.max_ctx = max_ctx;
    const cudaError_t e = iv2::launch_attn_split(qr, k, v, lcap, idx, cnt, mc, false, nullptr, nullptr, nullptr, out,
                                                 lse, scratch, (cudaStream_t)stream);
    return e == cudaSuccess ? INFLLMV2_OK : INFLLMV2_ERR_CUDA;
}

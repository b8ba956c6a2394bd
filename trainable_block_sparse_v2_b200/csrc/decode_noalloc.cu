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

}  // namespace

extern "C" int infllmv2_sparse_attn_decode_noalloc(const void* q, int batch, int hq, int hkv, int head_dim,
                                                   const void* k, const void* v, int lcap, const int32_t* ctx_lens,
                                                   int max_ctx, const int32_t* idx, const int32_t* cnt,
                                                   const infllmv2_params* params, void* out, float* lse,
                                                   infllmv2_stream_t stream)
{
    // the same argument checks as infllmv2_sparse_attn_decode
    iv2::MethodConsts mc;
    int nsplit = 0;
    const int st = iv2::check_decode_attn(q, batch, hq, hkv, head_dim, k, v, lcap, ctx_lens, max_ctx, idx, cnt, params,
                                          out, lse, &mc, &nsplit);
    if (st != INFLLMV2_OK) return st;
    // the partials of this call must fit the static array
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
    qr.cu_q = nullptr;
    qr.q_rows = batch;
    const cudaError_t e = iv2::launch_attn_split(qr, k, v, iv2::kv_contiguous(batch, lcap), idx, cnt, mc, false, nullptr, nullptr, nullptr, out,
                                                 lse, scratch, (cudaStream_t)stream);
    return e == cudaSuccess ? INFLLMV2_OK : INFLLMV2_ERR_CUDA;
}

// pool.cu -- semantic-kernel pooling (step 1 of InfLLM v2).
//
// kern[b, g, j, :] = bf16_rne( mean of k[b, i, g, :] over the 32-key window i in [16 j, 16 j + 32) )
// for the windows completed between old_lens[b] and new_lens[b] keys ("Tsinghua & ModelBest: MiniCPM4
// technical details", "Model architecture: InfLLM v2", item 1: every block is made of several
// fine-grained semantic kernels; the pages give no window size).
//
// HBM-bound: every key row is read once.  A window of 32 keys is the sum of two 16-key half windows
// that it shares with its neighbours, so each CTA first sums 33 half windows into shared memory and then
// forms 32 kernels from adjacent pairs.  Rows are 16-byte coalesced loads (d = 128: 16 lanes cover one
// 256-byte row), and all 16 rows of a half window are in flight per thread.
//
// Exactness.  The kernel is the window mean rounded ONCE to bf16.  The sums are formed in fp64: a bf16
// value has an 8-bit significand, so a sum of 32 of them is exact in fp64 unless their exponents spread
// over more than ~40 binary orders (never for activations of a model; an fp32 sum of N(0,1) keys is
// inexact about once in a few million kernels and then double-rounds).  The scaling by 1/32 is exact, and
// the fp64 mean reaches bf16 through one correctly rounded step: round-to-odd into fp32, then
// round-to-nearest-even into bf16.  Rounding to odd into a format with at least two more significand bits
// than the target makes the second rounding equal to a direct one (S. Boldo and G. Melquiond, "Emulation
// of FMA and correctly rounded sums: proved algorithms using rounding to odd", IEEE Trans. Computers 57(4),
// 2008); fp32 has 24 bits against bf16's 8.
#include "common.cuh"
#include "internal.h"

namespace iv2 {

constexpr int kPoolKernelsPerCta = 32;
constexpr int kPoolThreads = 256;

template <int D>
__global__ void __launch_bounds__(kPoolThreads) kernel_pool_kernel(const __nv_bfloat16* __restrict__ k, KvRows kr,
                                                                   int Hkv, const int32_t* __restrict__ old_lens,
                                                                   const int32_t* __restrict__ new_lens,
                                                                   __nv_bfloat16* __restrict__ kern, int nk_cap)
{
    pdl_launch_dependents();
    pdl_wait();
    constexpr int CH = D / 8;                  // 16-byte chunks per row
    constexpr int HALVES = kPoolKernelsPerCta + 1;
    __shared__ double hs[HALVES][D];  // exact half-window sums (33.8 KB at d = 128)

    const int bg = blockIdx.y;
    const int b = bg / Hkv, g = bg % Hkv;
    const int n_old = old_lens ? old_lens[b] : 0;
    const int n_new = new_lens ? new_lens[b] : kr.cu[b + 1] - kr.cu[b];
    const int j_begin = num_kernels(n_old) + blockIdx.x * kPoolKernelsPerCta;
    const int j_end = min(num_kernels(n_new), j_begin + kPoolKernelsPerCta);
    if (j_begin >= j_end || j_end > nk_cap) return;

    const size_t row_stride = (size_t)Hkv * D;
    const int n_halves = j_end - j_begin + 1;  // half windows j_begin .. j_end

    // half-window sums: item = (half h, chunk c)
    for (int item = threadIdx.x; item < n_halves * CH; item += kPoolThreads) {
        const int h = item / CH, c = item % CH;
        const int row0 = (j_begin + h) * kKernelStride;
        double acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0;
        uint4 buf[kKernelStride];
        // the 16 rows of a half window are consecutive in every layout (16 divides a 64-position page); a
        // page the table does not map reads as zeros
        const long r0 = kv_pos_row(kr, b, row0);
        const __nv_bfloat16* hr = k + (r0 * Hkv + g) * D + c * 8;
#pragma unroll
        for (int r = 0; r < kKernelStride; ++r)
            buf[r] = r0 >= 0 ? ld_nc_v4(hr + (size_t)r * row_stride) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int r = 0; r < kKernelStride; ++r) {
            const uint32_t w[4] = {buf[r].x, buf[r].y, buf[r].z, buf[r].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[2 * e] += (double)bf16_lo(w[e]);
                acc[2 * e + 1] += (double)bf16_hi(w[e]);
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) hs[h][c * 8 + e] = acc[e];
    }
    __syncthreads();

    constexpr double inv = 1.0 / kKernelSize;  // a power of two: the scaling is exact
    for (int item = threadIdx.x; item < (j_end - j_begin) * CH; item += kPoolThreads) {
        const int jj = item / CH, c = item % CH;
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const double lo = (hs[jj][c * 8 + 2 * e] + hs[jj + 1][c * 8 + 2 * e]) * inv;
            const double hi = (hs[jj][c * 8 + 2 * e + 1] + hs[jj + 1][c * 8 + 2 * e + 1]) * inv;
            w[e] = (uint32_t)f64_to_bf16_rne(lo) | ((uint32_t)f64_to_bf16_rne(hi) << 16);
        }
        __nv_bfloat16* dst = kern + (((size_t)b * Hkv + g) * nk_cap + j_begin + jj) * D + c * 8;
        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

cudaError_t launch_kernel_pool(const void* k, int B, const KvRows& kr, int Hkv, int D, const int32_t* old_lens,
                               const int32_t* new_lens, int max_new_keys, void* kern, int nk_cap, cudaStream_t s)
{
    // windows completed by appending max_new_keys keys: at most max_new_keys / 16 + 1
    const int max_new_kernels = max_new_keys / kKernelStride + 1;
    dim3 grid((max_new_kernels + kPoolKernelsPerCta - 1) / kPoolKernelsPerCta, B * Hkv);
    const auto* kp = static_cast<const __nv_bfloat16*>(k);
    auto* kn = static_cast<__nv_bfloat16*>(kern);
    if (D == 128)
        return launch_pdl(kernel_pool_kernel<128>, grid, dim3(kPoolThreads), 0, s, kp, kr, Hkv, old_lens, new_lens,
                          kn, nk_cap);
    return launch_pdl(kernel_pool_kernel<64>, grid, dim3(kPoolThreads), 0, s, kp, kr, Hkv, old_lens, new_lens, kn,
                      nk_cap);
}

// ---------------------------------------------------------------------------------------------------
// Gradient of the semantic kernels with respect to K (training; MiniCPM4 technical details, "Model
// architecture: InfLLM v2", item 3 -- the derivative of step 1's definition, the bf16 rounding of the kernels
// taken as the identity): the transpose of the window mean.  With windows of 32 keys at stride 16, the keys of
// the 16-key chunk c lie in exactly the windows c - 1 and c, so every key of the chunk receives
//   dk = (dkern[c - 1] + dkern[c]) / 32         (a term only for a window j in [0, nk(len)))
// fp32: the pair is summed with one rounding and the power-of-two scale is exact, so a normal result is the
// correctly rounded value of the exact one.  One CTA writes one chunk of one (sequence, KV head): 16 rows of
// d fp32 in 16-byte stores; the two kernel rows it reads are shared by all of them through L1.  Lengths are
// clamped to Lcap and the kernel index to nk_cap, so no device-side value can move an access out of bounds.
// ---------------------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) kernel_pool_bwd_kernel(const float4* __restrict__ dkern,
                                                             const int32_t* __restrict__ lens, int Lcap, int Hkv,
                                                             int nk_cap, float4* __restrict__ dk, int accumulate)
{
    pdl_launch_dependents();
    pdl_wait();
    constexpr int F = D / 4;  // float4 per row
    const int c = blockIdx.x;
    const int bg = blockIdx.y, b = bg / Hkv, g = bg % Hkv;
    const int len = min(lens[b], Lcap);
    const int i0 = c * kKernelStride;
    if (i0 >= len) return;
    const int nk = min(len >= kKernelSize ? (len - kKernelSize) / kKernelStride + 1 : 0, nk_cap);
    const bool has_a = c >= 1 && c - 1 < nk, has_b = c < nk;
    const float4* row_a = dkern + ((size_t)bg * nk_cap + (has_a ? c - 1 : 0)) * F;
    const float4* row_b = dkern + ((size_t)bg * nk_cap + (has_b ? c : 0)) * F;
    const int rows = min(kKernelStride, len - i0);
    constexpr float kInv = 1.f / kKernelSize;
    for (int e = threadIdx.x; e < rows * F; e += blockDim.x) {
        const int row = e / F, f = e % F;
        const float4 za = has_a ? row_a[f] : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 zb = has_b ? row_b[f] : make_float4(0.f, 0.f, 0.f, 0.f);
        float4 v = make_float4((za.x + zb.x) * kInv, (za.y + zb.y) * kInv, (za.z + zb.z) * kInv, (za.w + zb.w) * kInv);
        float4* dst = dk + (((size_t)b * Lcap + i0 + row) * Hkv + g) * F + f;
        if (accumulate) {
            const float4 o = *dst;
            v = make_float4(o.x + v.x, o.y + v.y, o.z + v.z, o.w + v.w);
        }
        *dst = v;
    }
}

cudaError_t launch_kernel_pool_backward(const float* dkern, int B, int Lcap, int Hkv, int D, const int32_t* lens,
                                        int max_len, int nk_cap, float* dk, bool accumulate, cudaStream_t s)
{
    const dim3 grid((max_len + kKernelStride - 1) / kKernelStride, B * Hkv);
    const auto* dkp = reinterpret_cast<const float4*>(dkern);
    auto* dkq = reinterpret_cast<float4*>(dk);
    if (D == 128)
        return launch_pdl(kernel_pool_bwd_kernel<128>, grid, dim3(128), 0, s, dkp, lens, Lcap, Hkv, nk_cap, dkq,
                          accumulate ? 1 : 0);
    return launch_pdl(kernel_pool_bwd_kernel<64>, grid, dim3(128), 0, s, dkp, lens, Lcap, Hkv, nk_cap, dkq,
                      accumulate ? 1 : 0);
}

// ---------------------------------------------------------------------------------------------------
// Cache maintenance of a decode step (the pages have no counterpart): one new key and value row per
// sequence into the caches, k_cache[b, pos[b], :, :] = k_new[b, :, :] (v likewise).  16-byte copies; a
// position outside [0, Lcap) writes nothing.  With a paged cache the row is that of position pos[b] through
// the page table, and a position past the table or on a page id outside [0, num_pages) writes nothing.
// ---------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) kv_append_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                                       const int32_t* __restrict__ pos, KvRows kr, int row16,
                                                       uint4* __restrict__ k_cache, uint4* __restrict__ v_cache)
{
    pdl_launch_dependents();
    pdl_wait();
    const int b = blockIdx.x;
    const int p = pos[b];
    if (p < 0 || (!kr.table && p >= kr.Lcap)) return;
    const long r = kv_pos_row(kr, b, p);
    if (r < 0) return;
    const size_t dst = (size_t)r * row16;
    for (int i = threadIdx.x; i < 2 * row16; i += blockDim.x) {
        if (i < row16) k_cache[dst + i] = k_new[(size_t)b * row16 + i];
        else v_cache[dst + i - row16] = v_new[(size_t)b * row16 + i - row16];
    }
}

cudaError_t launch_kv_append(const void* k_new, const void* v_new, int B, int Hkv, int D, const int32_t* pos,
                             void* k_cache, void* v_cache, const KvRows& kr, cudaStream_t s)
{
    const int row16 = Hkv * D / 8;  // 16-byte chunks of one position's keys (all KV heads)
    return launch_pdl(kv_append_kernel, dim3(B), dim3(256), 0, s, static_cast<const uint4*>(k_new),
                      static_cast<const uint4*>(v_new), pos, kr, row16, static_cast<uint4*>(k_cache),
                      static_cast<uint4*>(v_cache));
}

}  // namespace iv2

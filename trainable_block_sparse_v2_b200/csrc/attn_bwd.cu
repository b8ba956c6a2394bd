// attn_bwd.cu -- gradients of the block-sparse attention for a fixed selection (training).
//
// The pages train InfLLM v2 with the same sparse attention they run at inference ("Tsinghua & ModelBest:
// MiniCPM4 technical details", "Model architecture: InfLLM v2", item 3: efficient operators for training
// and inference) but print no backward; this is the derivative of the forward's definition.  The block
// selection is piecewise constant in q and K, so for a fixed selection the gradient flows only through the
// attention: for a row (token t, head h) with key set K(t), p_e = exp(scale q.k_e - lse),
//   dp_e = dout . v_e,  Dsum = dout . out,  ds_e = p_e (dp_e - Dsum)
//   dq   = scale sum_e ds_e k_e,   dk_e += scale ds_e q,   dv_e += p_e dout.
//
// Kernels, in stream order (each waits for the one before through programmatic dependent launch):
//  1. zero      dk, dv and the per-block counters;
//  2. prep      one warp per (token, group) row: Dsum of its heads, and one count per attended block;
//  3. scan      one CTA: exclusive scan of the counts (list offsets) and of the chunk counts (work items
//               of at most kItemTokens tokens of one block's list);
//  4. fill      one warp per row: writes the token into the list of every block it attends (the order
//               inside a list follows the atomics, so the fp32 sums of dk / dv are equal up to rounding
//               order from run to run);
//  4b. order    one CTA: the work items sorted by the first token of their chunk (a counting sort over
//               token buckets), so that the items the persistent dk / dv CTAs run at the same time gather
//               neighbouring tokens, whose Q and dO rows then come from L2 instead of DRAM;
//  5. dq        one warp per row, the forward's walk over the row's blocks in 32-key halves, double-
//               buffered (mma.sync m16n8k16 with the G <= 16 heads of the group as MMA rows):
//               S = Q K^T, P = 2^(S log2e - lse log2e), dP = dO V^T, dS = P (dP - Dsum), dQ += dS K;
//  6. dkdv      persistent CTAs over the work items: a CTA stages one block's K and V (64 keys), each warp
//               owns 16 keys as MMA rows, and for every token of the chunk computes S^T = K Q^T,
//               dP^T = V dO^T (heads as MMA columns), then dV += P^T dO and dK += dS^T Q; the chunk's
//               sums go to dk / dv by vector fp32 atomics.
// Key sets are those of the forward (attn.cu): a dense row reads blocks 0..c, a sparse row the valid
// entries of its list, clipped to the keys before n.
#include "attn_warp.cuh"
#include "common.cuh"
#include "internal.h"

namespace iv2 {

namespace {

constexpr int kBwdRowWarps = 4;   // rows per CTA of the prep and fill kernels
constexpr int kDqWarps = 2;       // rows per CTA of the dq kernel: 64 KB of staging, three CTAs per SM
constexpr int kDkvThreads = 128;  // 4 warps x 16 keys of one 64-key block
constexpr int kItemTokens = 256;  // tokens per dkdv work item
constexpr int kScanThreads = 1024;
constexpr int kOrderBuckets = 4096;  // token buckets of the work-item sort

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// blocks a row may attend: its list (kmax) or, dense, every block of a context up to dense_len keys
int bwd_max_per_row(int max_ctx, int kmax, int dense_len, bool dense_all)
{
    const int all = (max_ctx + kBlock - 1) / kBlock;
    if (dense_all) return all;
    const int dense_blocks = (min(max_ctx, dense_len) + kBlock - 1) / kBlock;
    return min(all, max(kmax, dense_blocks));
}

struct BwdWsLayout {
    size_t dsum, counts, offsets, cursor, nitems, item_list, item_start, order_list, order_start, tokens, end;
    int nl, nb, cap, max_items;
};

BwdWsLayout bwd_layout(int B, int T, int Hq, int Hkv, int max_ctx, int kmax, int dense_len, bool dense_all)
{
    BwdWsLayout w;
    w.nb = (max_ctx + kBlock - 1) / kBlock;
    w.nl = B * Hkv * w.nb;
    const long cap = (long)B * T * Hkv * bwd_max_per_row(max_ctx, kmax, dense_len, dense_all);
    w.cap = (int)min(cap, (long)INT32_MAX);
    w.max_items = (int)min((long)w.nl + cap / kItemTokens + 1, (long)INT32_MAX);
    size_t o = 0;
    w.dsum = o;       o += round256((size_t)B * T * Hq * 4);
    w.counts = o;     o += round256((size_t)w.nl * 4);
    w.offsets = o;    o += round256((size_t)w.nl * 4);
    w.cursor = o;     o += round256((size_t)w.nl * 4);
    w.nitems = o;     o += 256;
    w.item_list = o;  o += round256((size_t)w.max_items * 4);
    w.item_start = o; o += round256((size_t)w.max_items * 4);
    w.order_list = o; o += round256((size_t)w.max_items * 4);
    w.order_start = o; o += round256((size_t)w.max_items * 4);
    w.tokens = o;     o += round256((size_t)w.cap * 4);
    w.end = o;
    return w;
}

// ---------------------------------------------------------------------------------------------------
// 1. zero
// ---------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) bwd_zero_kernel(float4* __restrict__ a, size_t na, float4* __restrict__ b,
                                                       size_t nb, int* __restrict__ c, int nc)
{
    pdl_launch_dependents();
    pdl_wait();
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < na; i += stride) a[i] = z;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nb; i += stride) b[i] = z;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < (size_t)nc; i += stride) c[i] = 0;
}

// ---------------------------------------------------------------------------------------------------
// 2. prep: Dsum = dout . out per head, and the block counts
// ---------------------------------------------------------------------------------------------------
struct RowCtx {
    int g, t, b, G, n, c, count;
    long bt;
    bool dense;
    const int32_t* idx_row;
};

IV2_DEV RowCtx row_ctx(const QueryRows& qr, long row, const int32_t* idx, const int32_t* cnt, const MethodConsts& mc,
                       int dense_all)
{
    RowCtx r;
    r.g = (int)(row % qr.Hkv);
    r.bt = row / qr.Hkv;
    r.t = (int)(r.bt % qr.T);
    r.b = (int)(r.bt / qr.T);
    r.G = qr.Hq / qr.Hkv;
    r.n = query_ctx(qr, r.b, r.t);
    r.c = (r.n - 1) / kBlock;
    r.dense = dense_all || r.n <= mc.dense_len;
    r.count = r.dense ? r.c + 1 : min(cnt[row], mc.kmax);
    r.idx_row = idx ? idx + row * mc.kmax : nullptr;
    return r;
}

template <int D>
__global__ void __launch_bounds__(kBwdRowWarps * 32) bwd_prep_kernel(QueryRows qr, const int32_t* __restrict__ idx,
                                                                     const int32_t* __restrict__ cnt, MethodConsts mc,
                                                                     int dense_all, int nb,
                                                                     const __nv_bfloat16* __restrict__ out,
                                                                     const __nv_bfloat16* __restrict__ dout,
                                                                     float* __restrict__ dsum, int* __restrict__ counts)
{
    pdl_launch_dependents();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long row = (long)blockIdx.x * kBwdRowWarps + warp;
    if (row >= (long)qr.B * qr.T * qr.Hkv) return;
    const RowCtx r = row_ctx(qr, row, idx, cnt, mc, dense_all);
    constexpr int CH = D / 8;  // 16-byte chunks of a head row; 32 / CH heads per pass
    for (int h0 = 0; h0 < r.G; h0 += 32 / CH) {
        const int hh = h0 + lane / CH, ch = lane % CH;
        float acc = 0.f;
        if (hh < r.G) {
            const size_t off = ((size_t)r.bt * qr.Hq + r.g * r.G + hh) * D + ch * 8;
            const uint4 a = *reinterpret_cast<const uint4*>(out + off);
            const uint4 d = *reinterpret_cast<const uint4*>(dout + off);
            acc = bf16_lo(a.x) * bf16_lo(d.x) + bf16_hi(a.x) * bf16_hi(d.x) + bf16_lo(a.y) * bf16_lo(d.y) +
                  bf16_hi(a.y) * bf16_hi(d.y) + bf16_lo(a.z) * bf16_lo(d.z) + bf16_hi(a.z) * bf16_hi(d.z) +
                  bf16_lo(a.w) * bf16_lo(d.w) + bf16_hi(a.w) * bf16_hi(d.w);
        }
#pragma unroll
        for (int o = 1; o < CH; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (ch == 0 && hh < r.G) dsum[(size_t)r.bt * qr.Hq + r.g * r.G + hh] = acc;
    }
    int* cl = counts + ((size_t)r.b * qr.Hkv + r.g) * nb;
    for (int k = lane; k < r.count; k += 32) {
        const int blk = row_block(r.dense, r.c, r.idx_row, r.count, k, r.n);
        if (blk >= 0 && blk < nb) atomicAdd(&cl[blk], 1);  // n <= max_ctx keeps blk < nb
    }
}

// ---------------------------------------------------------------------------------------------------
// 3. scan: list offsets, and work items (list, first token) of at most kItemTokens tokens
// ---------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kScanThreads) bwd_scan_kernel(const int* __restrict__ counts, int nl,
                                                                int* __restrict__ offsets, int* __restrict__ cursor,
                                                                int* __restrict__ nitems, int* __restrict__ item_list,
                                                                int* __restrict__ item_start, int max_items)
{
    pdl_launch_dependents();
    pdl_wait();
    __shared__ int wt[32], wc[32];
    __shared__ int carry_t, carry_c;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        carry_t = 0;
        carry_c = 0;
    }
    __syncthreads();
    for (int base = 0; base < nl; base += kScanThreads) {
        const int l = base + threadIdx.x;
        const int ct = l < nl ? counts[l] : 0;
        const int cc = (ct + kItemTokens - 1) / kItemTokens;
        int it = ct, ic = cc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, it, o);
            const int z = __shfl_up_sync(0xffffffffu, ic, o);
            if (lane >= o) {
                it += y;
                ic += z;
            }
        }
        if (lane == 31) {
            wt[warp] = it;
            wc[warp] = ic;
        }
        __syncthreads();
        if (warp == 0) {
            const int a = wt[lane], c = wc[lane];
            int ia = a, ic2 = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, ia, o);
                const int z = __shfl_up_sync(0xffffffffu, ic2, o);
                if (lane >= o) {
                    ia += y;
                    ic2 += z;
                }
            }
            wt[lane] = ia - a;
            wc[lane] = ic2 - c;
        }
        __syncthreads();
        const int ex_t = carry_t + wt[warp] + it - ct;
        const int ex_c = carry_c + wc[warp] + ic - cc;
        if (l < nl) {
            offsets[l] = ex_t;
            cursor[l] = ex_t;
            for (int j = 0; j < cc && ex_c + j < max_items; ++j) {
                item_list[ex_c + j] = l;
                item_start[ex_c + j] = j * kItemTokens;
            }
        }
        __syncthreads();  // every thread has read carry_* and the warp sums
        if (threadIdx.x == kScanThreads - 1) {
            carry_t = ex_t + ct;
            carry_c = ex_c + cc;
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) *nitems = min(carry_c, max_items);
}

// ---------------------------------------------------------------------------------------------------
// 4. fill: token ids into the lists
// ---------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kBwdRowWarps * 32) bwd_fill_kernel(QueryRows qr, const int32_t* __restrict__ idx,
                                                                     const int32_t* __restrict__ cnt, MethodConsts mc,
                                                                     int dense_all, int nb, int* __restrict__ cursor,
                                                                     int* __restrict__ tokens, int cap)
{
    pdl_launch_dependents();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long row = (long)blockIdx.x * kBwdRowWarps + warp;
    if (row >= (long)qr.B * qr.T * qr.Hkv) return;
    const RowCtx r = row_ctx(qr, row, idx, cnt, mc, dense_all);
    int* cl = cursor + ((size_t)r.b * qr.Hkv + r.g) * nb;
    for (int k = lane; k < r.count; k += 32) {
        const int blk = row_block(r.dense, r.c, r.idx_row, r.count, k, r.n);
        if (blk < 0 || blk >= nb) continue;
        const int pos = atomicAdd(&cl[blk], 1);
        if (pos < cap) tokens[pos] = r.t;
    }
}

// ---------------------------------------------------------------------------------------------------
// 4b. order: a counting sort of the work items by (batch, first token of the chunk) >> shift, stable up to
// the order of the shared-memory atomics (any order of the items gives the same sums up to rounding order)
__global__ void __launch_bounds__(kScanThreads) bwd_order_kernel(const int* __restrict__ nitems,
                                                                 const int* __restrict__ item_list,
                                                                 const int* __restrict__ item_start,
                                                                 const int* __restrict__ offsets,
                                                                 const int* __restrict__ tokens, int cap,
                                                                 int lists_per_batch, int T, int shift,
                                                                 int* __restrict__ order_list,
                                                                 int* __restrict__ order_start)
{
    pdl_launch_dependents();
    pdl_wait();
    __shared__ int hist[kOrderBuckets];
    __shared__ int wsum[32];
    const int n = *nitems;
    for (int i = threadIdx.x; i < kOrderBuckets; i += kScanThreads) hist[i] = 0;
    __syncthreads();
    // the bucket of item i; the token read is clamped into the list array, and the bucket into the histogram
    // (a list entry past cap was never written: its value only orders the items)
    auto bucket = [&](int i) {
        const int l = item_list[i];
        const long at = max(0L, min((long)offsets[l] + item_start[i], (long)cap - 1));
        const long key = (long)(l / lists_per_batch) * T + (cap > 0 ? tokens[at] : 0);
        return (int)max(0L, min(key >> shift, (long)kOrderBuckets - 1));
    };
    for (int i = threadIdx.x; i < n; i += kScanThreads) atomicAdd(&hist[bucket(i)], 1);
    __syncthreads();
    // exclusive scan of the buckets, kOrderBuckets / kScanThreads consecutive ones per thread
    constexpr int kPer = kOrderBuckets / kScanThreads;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int c[kPer], tot = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        c[j] = hist[kPer * threadIdx.x + j];
        tot += c[j];
    }
    int incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int a = wsum[lane];
        int ia = a;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, ia, o);
            if (lane >= o) ia += y;
        }
        wsum[lane] = ia - a;
    }
    __syncthreads();
    int ex = wsum[warp] + incl - tot;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        hist[kPer * threadIdx.x + j] = ex;  // each thread rewrites only its own buckets
        ex += c[j];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kScanThreads) {
        const int slot = atomicAdd(&hist[bucket(i)], 1);
        order_list[slot] = item_list[i];
        order_start[slot] = item_start[i];
    }
}

// ---------------------------------------------------------------------------------------------------
// 5. dq: one warp per (token, group) row, over 32-key halves of its blocks (double-buffered per warp)
// ---------------------------------------------------------------------------------------------------
template <int D>
struct DqSmem {
    static constexpr int kHalf = 32 * D * 2;            // K or V rows of one 32-key half block
    static constexpr int kWarpBytes = 4 * kHalf;        // [2 buffers] x (K | V)
    static constexpr int kBytes = kDqWarps * kWarpBytes;
};

// stage rows [0, 32) of a half block: row r from src + r * row_stride when r < nvalid, else zeros
template <int D>
IV2_DEV void warp_load_half(unsigned char* dst, const __nv_bfloat16* src, size_t row_stride, int nvalid)
{
    constexpr int CH = D / 8;
    const int lane = threadIdx.x & 31;
#pragma unroll 4
    for (int i = lane; i < 32 * CH; i += 32) {
        const int r = i / CH, ch = i % CH;
        const bool ok = r < nvalid;
        cp_async_16_zfill(dst + swz_kv<D>(r, ch), src + (ok ? (size_t)r * row_stride : 0) + ch * 8, ok ? 16 : 0);
    }
}

// the next 32-key unit of a row after (kpos, half): returns the block (or -1) and updates kpos / half
IV2_DEV int next_half(const RowCtx& r, int& kpos, int& half)
{
    ++half;
    for (;;) {
        if (half == 2) {
            half = 0;
            ++kpos;
        }
        if (kpos >= r.count) return -1;
        const int blk = row_block(r.dense, r.c, r.idx_row, r.count, kpos, r.n);
        if (blk >= 0 && blk * kBlock + half * 32 < r.n) return blk;
        half = 2;  // invalid entry or a half past n: move to the next entry
    }
}

template <int D>
__global__ void __launch_bounds__(kDqWarps * 32) bwd_dq_kernel(QueryRows qr, const __nv_bfloat16* __restrict__ k,
                                                                   const __nv_bfloat16* __restrict__ v, int Lcap,
                                                                   const int32_t* __restrict__ idx,
                                                                   const int32_t* __restrict__ cnt, MethodConsts mc,
                                                                   int dense_all, const float* __restrict__ lse,
                                                                   const float* __restrict__ dsum,
                                                                   const __nv_bfloat16* __restrict__ dout,
                                                                   float* __restrict__ dq)
{
    using L = DqSmem<D>;
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ __align__(128) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
    const long row = (long)blockIdx.x * kDqWarps + warp;
    if (row >= (long)qr.B * qr.T * qr.Hkv) return;
    unsigned char* wsm = smem + warp * L::kWarpBytes;  // buffer u: K at u * 2 * kHalf, V right after
    const RowCtx r = row_ctx(qr, row, idx, cnt, mc, dense_all);
    const size_t head0 = (size_t)r.bt * qr.Hq + r.g * r.G;

    uint32_t qf[D / 16][4], df[D / 16][4];
    load_q_rows<D>(static_cast<const __nv_bfloat16*>(qr.q) + head0 * D, r.G, qf);
    load_q_rows<D>(dout + head0 * D, r.G, df);
    // per MMA row (head): lse in log2 units (+inf for padding rows: their p is 0) and Dsum
    float l2[2], dd[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int hr = gq + 8 * i;
        l2[i] = __int_as_float(0x7f800000);
        dd[i] = 0.f;
        if (hr < r.G) {
            const float lv = lse[head0 + hr];
            if (lv > neg_inf() && lv < __int_as_float(0x7f800000)) l2[i] = lv * kLog2e;
            dd[i] = dsum[head0 + hr];
        }
    }
    const size_t rs = (size_t)qr.Hkv * D;
    const __nv_bfloat16* kb = k + ((size_t)r.b * Lcap * qr.Hkv + r.g) * D;
    const __nv_bfloat16* vb = v + ((size_t)r.b * Lcap * qr.Hkv + r.g) * D;
    const float sl2 = mc.scale * kLog2e;
    float acc[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

    auto load_unit = [&](int blk, int half, int u) {
        const int key0 = blk * kBlock + half * 32;
        unsigned char* kd = wsm + u * 2 * L::kHalf;
        warp_load_half<D>(kd, kb + (size_t)key0 * rs, rs, min(32, r.n - key0));
        warp_load_half<D>(kd + L::kHalf, vb + (size_t)key0 * rs, rs, min(32, r.n - key0));
    };
    int kpos = 0, half = -1;
    int blk = next_half(r, kpos, half);
    if (blk >= 0) load_unit(blk, half, 0);
    cp_async_commit();
    int u = 0;
    while (blk >= 0) {
        int kpos2 = kpos, half2 = half;
        const int nblk = next_half(r, kpos2, half2);
        if (nblk >= 0) load_unit(nblk, half2, u ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncwarp();
        const unsigned char* ks_tile = wsm + u * 2 * L::kHalf;
        const unsigned char* vs_tile = ks_tile + L::kHalf;
        const int nvalid = r.n - (blk * kBlock + half * 32);  // keys of this unit before n (> 0)
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {  // 16 keys per step
            float s2[2][4], d2[2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                s2[j][0] = s2[j][1] = s2[j][2] = s2[j][3] = 0.f;
                d2[j][0] = d2[j][1] = d2[j][2] = d2[j][3] = 0.f;
                const int rr = (2 * kk + j) * 8 + (lane & 7);
#pragma unroll
                for (int ks = 0; ks < D / 16; ks += 2) {
                    const int ch = 2 * ks + (lane >> 3);
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4(b0, b1, b2, b3, ks_tile + swz_kv<D>(rr, ch));
                    mma_bf16_16816(s2[j], qf[ks], b0, b1);
                    mma_bf16_16816(s2[j], qf[ks + 1], b2, b3);
                    ldmatrix_x4(b0, b1, b2, b3, vs_tile + swz_kv<D>(rr, ch));
                    mma_bf16_16816(d2[j], df[ks], b0, b1);
                    mma_bf16_16816(d2[j], df[ks + 1], b2, b3);
                }
            }
            // P = 2^(S scale log2e - lse log2e) on keys before n, dS = P (dP - Dsum)
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int col = (2 * kk + j) * 8 + 2 * tq + (e & 1);
                    const float p = col < nvalid ? ex2_approx(s2[j][e] * sl2 - l2[e >> 1]) : 0.f;
                    s2[j][e] = p * (d2[j][e] - dd[e >> 1]);
                }
            uint32_t a[4];
            a[0] = pack_bf16(s2[0][0], s2[0][1]);
            a[1] = pack_bf16(s2[0][2], s2[0][3]);
            a[2] = pack_bf16(s2[1][0], s2[1][1]);
            a[3] = pack_bf16(s2[1][2], s2[1][3]);
            // dQ += dS K (K rows as the k16 x n8 operand, transposed by ldmatrix)
#pragma unroll
            for (int nd = 0; nd < D / 8; nd += 2) {
                const int mi = lane >> 3;
                const int rr = 16 * kk + (mi & 1) * 8 + (lane & 7);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(b0, b1, b2, b3, ks_tile + swz_kv<D>(rr, nd + (mi >> 1)));
                mma_bf16_16816(acc[nd], a, b0, b1);
                mma_bf16_16816(acc[nd + 1], a, b2, b3);
            }
        }
        __syncwarp();  // buffer u is read: the unit after next may land in it
        blk = nblk;
        kpos = kpos2;
        half = half2;
        u ^= 1;
    }
    cp_async_wait<0>();
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int hr = gq + 8 * i;
        if (hr >= r.G) continue;
        float* drow = dq + (head0 + hr) * D;
#pragma unroll
        for (int nd = 0; nd < D / 8; ++nd)
            *reinterpret_cast<float2*>(drow + nd * 8 + 2 * tq) =
                make_float2(acc[nd][2 * i] * mc.scale, acc[nd][2 * i + 1] * mc.scale);
    }
}

// ---------------------------------------------------------------------------------------------------
// 6. dk, dv: one block's keys against the tokens of its list
// ---------------------------------------------------------------------------------------------------
template <int D>
struct DkvSmem {
    static constexpr int kTile = kBlock * D * 2;     // K or V of the block
    static constexpr int kRows = 16 * D * 2;         // 16 head rows of q or dout
    static constexpr int kK = 0;
    static constexpr int kV = kTile;
    static constexpr int kStage = 2 * kTile;         // [2] x (q rows | dout rows)
    static constexpr int kStageBytes = 2 * kRows;
    static constexpr int kScal = kStage + 2 * kStageBytes;  // [2][16] lse2, [2][16] Dsum, [2] n
    static constexpr int kBytes = kScal + 4 * 16 * 4 + 16;
};

template <int D>
__global__ void __launch_bounds__(kDkvThreads) bwd_dkdv_kernel(QueryRows qr, const __nv_bfloat16* __restrict__ k,
                                                               const __nv_bfloat16* __restrict__ v, int Lcap,
                                                               MethodConsts mc, int nb, const float* __restrict__ lse,
                                                               const float* __restrict__ dsum,
                                                               const __nv_bfloat16* __restrict__ dout,
                                                               const int* __restrict__ counts,
                                                               const int* __restrict__ offsets,
                                                               const int* __restrict__ tokens,
                                                               const int* __restrict__ nitems,
                                                               const int* __restrict__ item_list,
                                                               const int* __restrict__ item_start, int cap,
                                                               float* __restrict__ dk, float* __restrict__ dv)
{
    using L = DkvSmem<D>;
    constexpr int CH = D / 8;
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
    const int G = qr.Hq / qr.Hkv;
    float* lse2_s = reinterpret_cast<float*>(smem + L::kScal);  // [2][16]
    float* dsum_s = lse2_s + 32;                                // [2][16]
    int* n_s = reinterpret_cast<int*>(dsum_s + 32);             // [2]
    const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(qr.q);
    const size_t rs = (size_t)qr.Hkv * D;
    const float sl2 = mc.scale * kLog2e;
    const int n_items = *nitems;

    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int l = item_list[item], start = item_start[item];
        const int b = l / (qr.Hkv * nb), g = (l / nb) % qr.Hkv, kb = l % nb;
        // (a list holds at most its row count of tokens; the clamp to the list storage only matters for
        // block lists with repeated ids, which the fill kernel drops past the storage)
        const int ntok = min(min(kItemTokens, counts[l] - start), cap - offsets[l] - start);
        if (ntok <= 0) continue;
        const int* toks = tokens + offsets[l] + start;
        // the block's K and V (rows past the cache read as zeros)
        const int nrows = min(kBlock, Lcap - kb * kBlock);
        const __nv_bfloat16* kbase = k + (((size_t)b * Lcap + (size_t)kb * kBlock) * qr.Hkv + g) * D;
        const __nv_bfloat16* vbase = v + (((size_t)b * Lcap + (size_t)kb * kBlock) * qr.Hkv + g) * D;
        for (int i = tid; i < kBlock * CH; i += kDkvThreads) {
            const int rr = i / CH, ch = i % CH;
            const bool ok = rr < nrows;
            cp_async_16_zfill(smem + L::kK + swz_kv<D>(rr, ch), kbase + (ok ? (size_t)rr * rs : 0) + ch * 8, ok ? 16 : 0);
            cp_async_16_zfill(smem + L::kV + swz_kv<D>(rr, ch), vbase + (ok ? (size_t)rr * rs : 0) + ch * 8, ok ? 16 : 0);
        }
        // q and dout rows of token j (heads past G read as zeros; their lse2 is +inf, so their p is 0)
        auto stage = [&](int j, int buf) {
            const int t = toks[j];
            const size_t head0 = ((size_t)b * qr.T + t) * qr.Hq + (size_t)g * G;
            unsigned char* qs = smem + L::kStage + buf * L::kStageBytes;
            unsigned char* ds = qs + L::kRows;
            for (int i = tid; i < 16 * CH; i += kDkvThreads) {
                const int rr = i / CH, ch = i % CH;
                const bool ok = rr < G;
                const size_t off = (head0 + (ok ? rr : 0)) * D + ch * 8;
                cp_async_16_zfill(qs + swz_kv<D>(rr, ch), qg + off, ok ? 16 : 0);
                cp_async_16_zfill(ds + swz_kv<D>(rr, ch), dout + off, ok ? 16 : 0);
            }
            if (tid < 16) {
                float l2 = __int_as_float(0x7f800000), dd = 0.f;
                if (tid < G) {
                    const float lv = lse[head0 + tid];
                    if (lv > neg_inf() && lv < __int_as_float(0x7f800000)) l2 = lv * kLog2e;
                    dd = dsum[head0 + tid];
                }
                lse2_s[buf * 16 + tid] = l2;
                dsum_s[buf * 16 + tid] = dd;
            }
            if (tid == 0) n_s[buf] = query_ctx(qr, b, t);
        };

        float ak[D / 8][4], av[D / 8][4];
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            ak[i][0] = ak[i][1] = ak[i][2] = ak[i][3] = 0.f;
            av[i][0] = av[i][1] = av[i][2] = av[i][3] = 0.f;
        }
        stage(0, 0);
        cp_async_commit();
        const int key0 = kb * kBlock + 16 * warp + gq;  // this lane's MMA rows: keys key0, key0 + 8
        for (int j = 0; j < ntok; ++j) {
            const int buf = j & 1;
            if (j + 1 < ntok) stage(j + 1, buf ^ 1);
            cp_async_commit();
            cp_async_wait<1>();
            __syncthreads();
            const unsigned char* qs = smem + L::kStage + buf * L::kStageBytes;
            const unsigned char* ds = qs + L::kRows;
            const float* l2 = lse2_s + buf * 16;
            const float* dd = dsum_s + buf * 16;
            const int n_tok = n_s[buf];
            // S^T = K Q^T and dP^T = V dO^T: 16 keys x 16 heads
            float st[2][4], dpt[2][4];
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int e = 0; e < 4; ++e) st[i][e] = dpt[i][e] = 0.f;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const int ar = 16 * warp + (lane & 15), ach = 2 * ks + (lane >> 4);
                const int br = (lane & 7) + 8 * (lane >> 4), bch = 2 * ks + ((lane >> 3) & 1);
                uint32_t a[4], b0, b1, b2, b3;
                ldmatrix_x4(a[0], a[1], a[2], a[3], smem + L::kK + swz_kv<D>(ar, ach));
                ldmatrix_x4(b0, b1, b2, b3, qs + swz_kv<D>(br, bch));
                mma_bf16_16816(st[0], a, b0, b1);
                mma_bf16_16816(st[1], a, b2, b3);
                ldmatrix_x4(a[0], a[1], a[2], a[3], smem + L::kV + swz_kv<D>(ar, ach));
                ldmatrix_x4(b0, b1, b2, b3, ds + swz_kv<D>(br, bch));
                mma_bf16_16816(dpt[0], a, b0, b1);
                mma_bf16_16816(dpt[1], a, b2, b3);
            }
            // P^T and dS^T (C layout: rows = keys key0 (+8), cols = heads 8 nt + 2 tq (+1))
            float p[2][4], sd[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = key0 + 8 * (e >> 1);
                    const int h = nt * 8 + 2 * tq + (e & 1);
                    const float pv = key < n_tok ? ex2_approx(st[nt][e] * sl2 - l2[h]) : 0.f;
                    p[nt][e] = pv;
                    sd[nt][e] = pv * (dpt[nt][e] - dd[h]);
                }
            const uint32_t pa[4] = {pack_bf16(p[0][0], p[0][1]), pack_bf16(p[0][2], p[0][3]),
                                    pack_bf16(p[1][0], p[1][1]), pack_bf16(p[1][2], p[1][3])};
            const uint32_t sa[4] = {pack_bf16(sd[0][0], sd[0][1]), pack_bf16(sd[0][2], sd[0][3]),
                                    pack_bf16(sd[1][0], sd[1][1]), pack_bf16(sd[1][2], sd[1][3])};
            // dV += P^T dO and dK += dS^T Q (head rows as the k16 x n8 operand, transposed by ldmatrix)
#pragma unroll
            for (int nd = 0; nd < D / 8; nd += 2) {
                const int mi = lane >> 3;
                const int rr = (mi & 1) * 8 + (lane & 7), ch = nd + (mi >> 1);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(b0, b1, b2, b3, ds + swz_kv<D>(rr, ch));
                mma_bf16_16816(av[nd], pa, b0, b1);
                mma_bf16_16816(av[nd + 1], pa, b2, b3);
                ldmatrix_x4_trans(b0, b1, b2, b3, qs + swz_kv<D>(rr, ch));
                mma_bf16_16816(ak[nd], sa, b0, b1);
                mma_bf16_16816(ak[nd + 1], sa, b2, b3);
            }
            __syncthreads();  // stage buf is free for token j + 2
        }
        cp_async_wait<0>();
        // this chunk's sums into dk, dv (keys past the cache have none)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int key = key0 + 8 * i;
            if (key >= Lcap) continue;
            const size_t base = (((size_t)b * Lcap + key) * qr.Hkv + g) * D + 2 * tq;
#pragma unroll
            for (int nd = 0; nd < D / 8; ++nd) {
                atomicAdd(reinterpret_cast<float2*>(dk + base + nd * 8),
                          make_float2(ak[nd][2 * i] * mc.scale, ak[nd][2 * i + 1] * mc.scale));
                atomicAdd(reinterpret_cast<float2*>(dv + base + nd * 8), make_float2(av[nd][2 * i], av[nd][2 * i + 1]));
            }
        }
        __syncthreads();  // tiles and stages free for the next item
    }
}

template <int D>
cudaError_t bwd_impl(const QueryRows& qr, const void* k, const void* v, int Lcap, const int32_t* idx,
                     const int32_t* cnt, const MethodConsts& mc, bool dense_all, const void* out, const float* lse,
                     const void* dout, float* dq, float* dk, float* dv, void* ws, cudaStream_t s)
{
    const BwdWsLayout w = bwd_layout(qr.B, qr.T, qr.Hq, qr.Hkv, qr.max_ctx, mc.kmax, mc.dense_len, dense_all);
    unsigned char* base = static_cast<unsigned char*>(ws);
    float* dsum = reinterpret_cast<float*>(base + w.dsum);
    int* counts = reinterpret_cast<int*>(base + w.counts);
    int* offsets = reinterpret_cast<int*>(base + w.offsets);
    int* cursor = reinterpret_cast<int*>(base + w.cursor);
    int* nitems = reinterpret_cast<int*>(base + w.nitems);
    int* item_list = reinterpret_cast<int*>(base + w.item_list);
    int* item_start = reinterpret_cast<int*>(base + w.item_start);
    int* order_list = reinterpret_cast<int*>(base + w.order_list);
    int* order_start = reinterpret_cast<int*>(base + w.order_start);
    int* tokens = reinterpret_cast<int*>(base + w.tokens);
    const int dense_flag = dense_all ? 1 : 0;
    const long rows = (long)qr.B * qr.T * qr.Hkv;
    const unsigned row_grid = (unsigned)((rows + kBwdRowWarps - 1) / kBwdRowWarps);
    const size_t nkv4 = (size_t)qr.B * Lcap * qr.Hkv * D / 4;

    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);

    cudaError_t e = launch_pdl(bwd_zero_kernel, dim3(4 * nsm), dim3(256), 0, s, reinterpret_cast<float4*>(dk), nkv4,
                               reinterpret_cast<float4*>(dv), nkv4, counts, w.nl);
    if (e != cudaSuccess) return e;
    e = launch_pdl(bwd_prep_kernel<D>, dim3(row_grid), dim3(kBwdRowWarps * 32), 0, s, qr, idx, cnt, mc, dense_flag,
                   w.nb, static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), dsum, counts);
    if (e != cudaSuccess) return e;
    e = launch_pdl(bwd_scan_kernel, dim3(1), dim3(kScanThreads), 0, s, static_cast<const int*>(counts), w.nl, offsets,
                   cursor, nitems, item_list, item_start, w.max_items);
    if (e != cudaSuccess) return e;
    e = launch_pdl(bwd_fill_kernel, dim3(row_grid), dim3(kBwdRowWarps * 32), 0, s, qr, idx, cnt, mc, dense_flag, w.nb,
                   cursor, tokens, w.cap);
    if (e != cudaSuccess) return e;
    int shift = 0;
    while (((long)qr.B * qr.T >> shift) >= kOrderBuckets) ++shift;
    e = launch_pdl(bwd_order_kernel, dim3(1), dim3(kScanThreads), 0, s, static_cast<const int*>(nitems),
                   static_cast<const int*>(item_list), static_cast<const int*>(item_start),
                   static_cast<const int*>(offsets), static_cast<const int*>(tokens), w.cap, qr.Hkv * w.nb, qr.T,
                   shift, order_list, order_start);
    if (e != cudaSuccess) return e;
    e = cudaErrorNotSupported;
    if (D == 128 && bwd_dq_tc_supported(qr))
        e = launch_bwd_dq_tc(qr, k, v, Lcap, idx, cnt, mc, dense_all, lse, dsum, dout, dq, s);
    if (e == cudaErrorNotSupported) {  // other shapes: the mma.sync kernel
        const size_t dq_smem = (size_t)DqSmem<D>::kBytes;
        e = ensure_smem(bwd_dq_kernel<D>, dq_smem);
        if (e != cudaSuccess) return e;
        const unsigned dq_grid = (unsigned)((rows + kDqWarps - 1) / kDqWarps);
        e = launch_pdl(bwd_dq_kernel<D>, dim3(dq_grid), dim3(kDqWarps * 32), dq_smem, s, qr,
                       static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), Lcap, idx, cnt, mc,
                       dense_flag, lse, static_cast<const float*>(dsum), static_cast<const __nv_bfloat16*>(dout), dq);
    }
    if (e != cudaSuccess) return e;
    if (D == 128 && bwd_dkdv_tc_supported(qr)) {
        e = launch_bwd_dkdv_tc(qr, k, v, Lcap, mc, w.nb, lse, dsum, dout, counts, offsets, tokens, nitems, order_list,
                               order_start, w.cap, w.max_items, dk, dv, s);
        if (e != cudaErrorNotSupported) return e;
    }
    e = ensure_smem(bwd_dkdv_kernel<D>, DkvSmem<D>::kBytes);
    if (e != cudaSuccess) return e;
    int per_sm = 1;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, bwd_dkdv_kernel<D>, kDkvThreads, DkvSmem<D>::kBytes);
    const int grid = (int)min((long)max(per_sm, 1) * nsm, (long)w.max_items);
    return launch_pdl(bwd_dkdv_kernel<D>, dim3(grid), dim3(kDkvThreads), (size_t)DkvSmem<D>::kBytes, s, qr,
                      static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), Lcap, mc, w.nb, lse,
                      static_cast<const float*>(dsum), static_cast<const __nv_bfloat16*>(dout),
                      static_cast<const int*>(counts), static_cast<const int*>(offsets),
                      static_cast<const int*>(tokens), static_cast<const int*>(nitems),
                      static_cast<const int*>(order_list), static_cast<const int*>(order_start), w.cap, dk, dv);
}

}  // namespace

size_t attn_bwd_ws_bytes(int B, int T, int Hq, int Hkv, int max_ctx, int kmax, int dense_len, bool dense_all)
{
    return bwd_layout(B, T, Hq, Hkv, max_ctx, kmax, dense_len, dense_all).end;
}

cudaError_t launch_attn_backward(const QueryRows& qr, const void* k, const void* v, int Lcap, const int32_t* idx,
                                 const int32_t* cnt, const MethodConsts& mc, bool dense_all, const void* out,
                                 const float* lse, const void* dout, float* dq, float* dk, float* dv, void* ws,
                                 cudaStream_t s)
{
    return qr.D == 128 ? bwd_impl<128>(qr, k, v, Lcap, idx, cnt, mc, dense_all, out, lse, dout, dq, dk, dv, ws, s)
                       : bwd_impl<64>(qr, k, v, Lcap, idx, cnt, mc, dense_all, out, lse, dout, dq, dk, dv, ws, s);
}

}  // namespace iv2

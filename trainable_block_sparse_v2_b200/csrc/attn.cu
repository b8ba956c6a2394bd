// attn.cu -- block-sparse attention over the selected blocks (step 3 of InfLLM v2), mma.sync path.
//
// Query (b, t), head h of group g, context n (MiniCPM4 technical details, InfLLM v2 overview: only the
// selected context blocks take part in attention; launch article section 1: short contexts dense):
//   keys = [0, n) when dense, else U_{blk in idx} [64 blk, min(64 blk + 64, n))
//   out  = sum_i softmax_i(scale q.k_i) v_i,   lse = log sum_i exp(scale q.k_i)
// Tree verification adds the draft keys whose bit is set in the query's bit-packed ancestor mask
// (QbitAI article, "speculative sampling, quantisation and long text", long-context bullet).
//
// One warp owns the 16 MMA rows of one query token: the G heads of its group (the heads share the block
// set, so they share every K/V tile -- item 2 of "Model architecture: InfLLM v2" is what makes the tile
// dense).  A 64-key block is staged in shared memory with cp.async (swizzled 16-byte chunks so ldmatrix
// is conflict-free), S = Q K^T and O += P V run on m16n8k16, and the softmax is the online (running max
// / running sum) form in log2 units.
//  * prefill: one warp per (token, group) row walks the row's whole block list.
//  * decode / tree: the block list of a row is split across CTAs (4 blocks per CTA, one per warp); each
//    CTA merges its warps and writes (max, sum, unnormalised O) to the workspace; a merge kernel (one CTA
//    per row and head) combines the splits by their LSE.  Tree rows get one extra split that attends to
//    the draft tile.
#include "attn_warp.cuh"
#include "common.cuh"
#include "internal.h"

namespace iv2 {

// =====================================================================================================
// prefill: one warp per (token, group) row
// =====================================================================================================
constexpr int kRowWarps = 4;

template <int D>
__global__ void __launch_bounds__(kRowWarps * 32) attn_rows_kernel(QueryRows qr, const __nv_bfloat16* __restrict__ k,
                                                                   const __nv_bfloat16* __restrict__ v, KvRows kr,
                                                                   const int32_t* __restrict__ idx,
                                                                   const int32_t* __restrict__ cnt, MethodConsts mc,
                                                                   int dense_all, __nv_bfloat16* __restrict__ out,
                                                                   float* __restrict__ lse)
{
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ __align__(128) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
    const long row = (long)blockIdx.x * kRowWarps + warp;
    const int rows = qr.B * qr.T * qr.Hkv;
    if (row >= rows) return;
    unsigned char* ks_tile = smem + warp * 2 * KvTile<D>::kBytes;
    unsigned char* vs_tile = ks_tile + KvTile<D>::kBytes;

    const int g = (int)(row % qr.Hkv);
    const int t = (int)((row / qr.Hkv) % qr.T), b = (int)(row / qr.Hkv / qr.T);
    if (t >= q_len(qr, b)) return;           // past this sequence's queries (packed batch)
    const long bt = q_row(qr, b, t);         // row of q / out / lse
    const long orow_i = bt * qr.Hkv + g;     // row of idx / cnt
    const int G = qr.Hq / qr.Hkv;
    const int n = query_ctx(qr, b, t);
    const int c = (n - 1) / kBlock;
    const bool dense = dense_all || n <= mc.dense_len;
    const int count = dense ? c + 1 : min(cnt[orow_i], mc.kmax);
    const int32_t* idx_row = idx ? idx + orow_i * mc.kmax : nullptr;

    uint32_t qf[D / 16][4];
    load_q_rows<D>(static_cast<const __nv_bfloat16*>(qr.q) + ((size_t)bt * qr.Hq + g * G) * D, G, qf);
    const size_t rs = (size_t)qr.Hkv * D;
    const float sl2 = mc.scale * kLog2e;
    // first key (value) row of block blk and the keys to stage from it (0 for a page the table does not map)
    auto block_src = [&](const __nv_bfloat16* base, int blk, int& nv) {
        const long r0 = kv_block_row(kr, b, blk);
        nv = r0 < 0 ? 0 : min(kBlock, n - blk * kBlock);
        return base + ((size_t)(r0 < 0 ? 0 : r0) * qr.Hkv + g) * D;
    };

    WarpAttnState<D> st;
    st.init();
    // first valid block
    int kpos = 0, blk = -1;
    while (kpos < count && (blk = row_block(dense, c, idx_row, count, kpos, n)) < 0) ++kpos;
    if (blk >= 0) {
        int nv;
        const __nv_bfloat16* ksrc = block_src(k, blk, nv);
        warp_load_tile<D>(ks_tile, ksrc, rs, nv);
        cp_async_commit();
        warp_load_tile<D>(vs_tile, block_src(v, blk, nv), rs, nv);
        cp_async_commit();
    }
    while (blk >= 0) {
        int knext = kpos + 1, nblk = -1;
        while (knext < count && (nblk = row_block(dense, c, idx_row, count, knext, n)) < 0) ++knext;
        cp_async_wait<1>();  // K of blk
        __syncwarp();
        float acc[8][4];
        tile_qk<D>(qf, ks_tile, acc);
        scale_mask(acc, sl2, prefix_mask64(n - blk * kBlock));
        __syncwarp();
        if (nblk >= 0) {
            int nv;
            const __nv_bfloat16* ksrc = block_src(k, nblk, nv);
            warp_load_tile<D>(ks_tile, ksrc, rs, nv);
        }
        cp_async_commit();
        cp_async_wait<1>();  // V of blk
        __syncwarp();
        tile_softmax_pv<D>(st, acc, vs_tile);
        __syncwarp();
        if (nblk >= 0) {
            int nv;
            const __nv_bfloat16* vsrc = block_src(v, nblk, nv);
            warp_load_tile<D>(vs_tile, vsrc, rs, nv);
        }
        cp_async_commit();
        blk = nblk;
        kpos = knext;
    }
    cp_async_wait<0>();
    finalize_rows<D>(st);

    // write rows gq, gq+8 (heads < G)
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int r = gq + 8 * i;
        if (r >= G) continue;
        const float inv = st.l[i] > 0.f ? 1.f / st.l[i] : 0.f;
        __nv_bfloat16* orow = out + ((size_t)bt * qr.Hq + g * G + r) * D;
#pragma unroll
        for (int nd = 0; nd < D / 8; ++nd)
            *reinterpret_cast<uint32_t*>(orow + nd * 8 + 2 * tq) =
                pack_bf16(st.o[nd][2 * i] * inv, st.o[nd][2 * i + 1] * inv);
        if (lse && tq == 0)
            lse[(size_t)bt * qr.Hq + g * G + r] = st.l[i] > 0.f ? (st.m[i] + __log2f(st.l[i])) * kLn2 : neg_inf();
    }
}

// =====================================================================================================
// decode / tree: split over the block list, merged by LSE
// =====================================================================================================
constexpr int kSplitWarps = 4;

int attn_split_count(int max_blocks) { return (max_blocks + kSplitWarps - 1) / kSplitWarps; }

int attn_split_max_blocks(int max_ctx, int kmax, int dense_len, bool dense_all, int window)
{
    const int all_blocks = (max_ctx + kBlock - 1) / kBlock;
    // a window of W keys starting anywhere touches at most ceil(W / 64) + 1 blocks
    if (window > 0) return min(all_blocks, (window + kBlock - 1) / kBlock + 1);
    if (dense_all) return all_blocks;
    const int dense_blocks = (min(max_ctx, dense_len) + kBlock - 1) / kBlock;
    return min(all_blocks, max(kmax, dense_blocks));
}

template <int D>
struct SplitWs {
    static constexpr int kFloats = 16 * D + 32;  // O[16][D], m[16], l[16]
};

size_t attn_ws_bytes(int rows, int nsplit)
{
    return ((size_t)rows * nsplit * SplitWs<128>::kFloats * 4 + 255) / 256 * 256;
}

template <int D>
__global__ void __launch_bounds__(kSplitWarps * 32) attn_split_kernel(
    QueryRows qr, const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v, KvRows kr,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt, MethodConsts mc, int dense_all, int nsplit_blocks,
    const __nv_bfloat16* __restrict__ k_draft, const __nv_bfloat16* __restrict__ v_draft,
    const uint32_t* __restrict__ tree_mask, float* __restrict__ ws)
{
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ __align__(128) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
    const int row = blockIdx.y;
    const int split = blockIdx.x;
    const int nsplit_total = gridDim.x;
    unsigned char* ks_tile = smem + warp * 2 * KvTile<D>::kBytes;
    unsigned char* vs_tile = ks_tile + KvTile<D>::kBytes;

    const int g = row % qr.Hkv, bt = row / qr.Hkv, t = bt % qr.T, b = bt / qr.T;
    const int G = qr.Hq / qr.Hkv;
    const int n = query_ctx(qr, b, t);
    const int c = (n - 1) / kBlock;
    const bool dense = dense_all || n <= mc.dense_len;
    // sliding window: the blocks of keys [w0, n), walked like a dense row from block w0 / 64
    const int w0 = mc.window > 0 ? max(0, n - mc.window) : 0;
    const int bw = w0 / kBlock;
    const int count = mc.window > 0 ? c + 1 - bw : (dense ? c + 1 : min(cnt[row], mc.kmax));
    const int32_t* idx_row = idx ? idx + (size_t)row * mc.kmax : nullptr;
    const float sl2 = mc.scale * kLog2e;

    const bool draft_split = tree_mask != nullptr && split == nsplit_blocks;
    if (!draft_split && split * kSplitWarps >= count) return;  // no block for this CTA: the merge skips it
    WarpAttnState<D> st;
    st.init();
    int blk = -1;
    bool work = false;
    uint64_t valid = 0;
    if (draft_split) {
        if (warp == 0) {
            // draft keys j < T of this sequence, visible when bit j of the node's mask is set
            const uint32_t msk = tree_mask[bt];
            valid = (uint64_t)msk & prefix_mask64(qr.T);
            const size_t rs = (size_t)qr.Hkv * D;
            const size_t base = ((size_t)b * qr.T * qr.Hkv + g) * D;
            warp_load_tile<D>(ks_tile, k_draft + base, rs, qr.T);
            warp_load_tile<D>(vs_tile, v_draft + base, rs, qr.T);
            cp_async_commit();
            work = true;
        }
    } else {
        const int e = split * kSplitWarps + warp;
        blk = mc.window > 0 ? (e < count ? bw + e : -1) : row_block(dense, c, idx_row, count, e, n);
        if (blk >= 0) {
            const size_t rs = (size_t)qr.Hkv * D;
            const long r0 = kv_block_row(kr, b, blk);  // -1: a page the table does not map (read as zeros)
            const size_t base = ((size_t)(r0 < 0 ? 0 : r0) * qr.Hkv + g) * D;
            const int nvalid = r0 < 0 ? 0 : min(kBlock, n - blk * kBlock);
            warp_load_tile<D>(ks_tile, k + base, rs, nvalid);
            warp_load_tile<D>(vs_tile, v + base, rs, nvalid);
            cp_async_commit();
            // keys [blk 64, blk 64 + nvalid), less those before the window's first key
            valid = prefix_mask64(nvalid) & ~prefix_mask64(max(0, w0 - blk * kBlock));
            work = true;
        }
    }
    if (work) {
        uint32_t qf[D / 16][4];
        load_q_rows<D>(static_cast<const __nv_bfloat16*>(qr.q) + ((size_t)bt * qr.Hq + g * G) * D, G, qf);
        cp_async_wait<0>();
        __syncwarp();
        float acc[8][4];
        tile_qk<D>(qf, ks_tile, acc);
        scale_mask(acc, sl2, valid);
        tile_softmax_pv<D>(st, acc, vs_tile);
        finalize_rows<D>(st);
    }
    __syncthreads();  // tiles are dead: reuse shared memory for the CTA merge

    // per-warp results to shared memory: O [warp][16][D], m/l [warp][16]
    float* so = reinterpret_cast<float*>(smem);
    float* sm = so + kSplitWarps * 16 * D;
    float* sl = sm + kSplitWarps * 16;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int r = gq + 8 * i;
#pragma unroll
        for (int nd = 0; nd < D / 8; ++nd) {
            so[(warp * 16 + r) * D + nd * 8 + 2 * tq] = st.o[nd][2 * i];
            so[(warp * 16 + r) * D + nd * 8 + 2 * tq + 1] = st.o[nd][2 * i + 1];
        }
        if (tq == 0) {
            sm[warp * 16 + r] = work ? st.m[i] : neg_inf();
            sl[warp * 16 + r] = work ? st.l[i] : 0.f;
        }
    }
    __syncthreads();
    float* wsp = ws + ((size_t)row * nsplit_total + split) * SplitWs<D>::kFloats;
    for (int item = threadIdx.x; item < G * D; item += kSplitWarps * 32) {
        const int r = item / D, d = item % D;
        float M = neg_inf();
#pragma unroll
        for (int w = 0; w < kSplitWarps; ++w) M = fmaxf(M, sm[w * 16 + r]);
        float O = 0.f, L = 0.f;
        if (M != neg_inf()) {
#pragma unroll
            for (int w = 0; w < kSplitWarps; ++w) {
                const float f = exp2_fast(sm[w * 16 + r] - M);
                O += so[(w * 16 + r) * D + d] * f;
                L += sl[w * 16 + r] * f;
            }
        }
        wsp[r * D + d] = O;
        if (d == 0) {
            wsp[16 * D + r] = M;
            wsp[16 * D + 16 + r] = L;
        }
    }
}

// one CTA per (row, head); thread d owns output column d.  Only the splits that received blocks (and the
// draft split of a tree row) are read.
template <int D>
__global__ void __launch_bounds__(D) attn_merge_kernel(QueryRows qr, const int32_t* __restrict__ cnt, MethodConsts mc,
                                                       int dense_all, int nsplit_blocks, int has_draft,
                                                       const float* __restrict__ ws, __nv_bfloat16* __restrict__ out,
                                                       float* __restrict__ lse)
{
    pdl_launch_dependents();
    pdl_wait();
    constexpr int kMaxSplits = 1024;
    __shared__ float fac[kMaxSplits];
    __shared__ float red[D / 32];
    const int row = blockIdx.x, r = blockIdx.y;
    const int g = row % qr.Hkv, bt = row / qr.Hkv, t = bt % qr.T, b = bt / qr.T;
    const int G = qr.Hq / qr.Hkv;
    const int n = query_ctx(qr, b, t);
    const int c = (n - 1) / kBlock;
    const bool dense = dense_all || n <= mc.dense_len;
    const int count = mc.window > 0 ? c + 1 - max(0, n - mc.window) / kBlock
                                    : (dense ? c + 1 : min(cnt[row], mc.kmax));
    const int nused = min((count + kSplitWarps - 1) / kSplitWarps, nsplit_blocks);
    const int nsplit_total = nsplit_blocks + has_draft;
    const float* base = ws + (size_t)row * nsplit_total * SplitWs<D>::kFloats;
    auto split_of = [&](int i) { return i < nused ? i : nsplit_blocks; };  // the draft split comes last
    const int nread = min(nused + has_draft, kMaxSplits);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    float m_loc = neg_inf();
    for (int i = threadIdx.x; i < nread; i += D) {
        const float m = base[(size_t)split_of(i) * SplitWs<D>::kFloats + 16 * D + r];
        fac[i] = m;
        m_loc = fmaxf(m_loc, m);
    }
    m_loc = warp_max(m_loc);
    if (lane == 0) red[warp] = m_loc;
    __syncthreads();
    float M = neg_inf();
#pragma unroll
    for (int w = 0; w < D / 32; ++w) M = fmaxf(M, red[w]);
    __syncthreads();
    float l_loc = 0.f;
    for (int i = threadIdx.x; i < nread; i += D) {
        const float f = (M == neg_inf()) ? 0.f : exp2_fast(fac[i] - M);
        fac[i] = f;
        l_loc += f * base[(size_t)split_of(i) * SplitWs<D>::kFloats + 16 * D + 16 + r];
    }
    l_loc = warp_sum(l_loc);
    __syncthreads();
    if (lane == 0) red[warp] = l_loc;
    __syncthreads();
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < D / 32; ++w) L += red[w];
    const int d = threadIdx.x;
    float O = 0.f;
#pragma unroll 8
    for (int i = 0; i < nread; ++i) O += fac[i] * base[(size_t)split_of(i) * SplitWs<D>::kFloats + r * D + d];
    out[((size_t)bt * qr.Hq + g * G + r) * D + d] = __float2bfloat16_rn(L > 0.f ? O / L : 0.f);
    if (lse && d == 0) lse[(size_t)bt * qr.Hq + g * G + r] = L > 0.f ? (M + __log2f(L)) * kLn2 : neg_inf();
}

// =====================================================================================================
// host side
// =====================================================================================================
template <int D>
static cudaError_t rows_impl(const QueryRows& qr, const void* k, const void* v, const KvRows& kr, const int32_t* idx,
                             const int32_t* cnt, const MethodConsts& mc, bool dense_all, void* out, float* lse,
                             cudaStream_t s)
{
    const size_t smem = (size_t)kRowWarps * 2 * KvTile<D>::kBytes;
    cudaError_t e = ensure_smem(attn_rows_kernel<D>, smem);
    if (e != cudaSuccess) return e;
    const long rows = (long)qr.B * qr.T * qr.Hkv;
    const unsigned grid = (unsigned)((rows + kRowWarps - 1) / kRowWarps);
    return launch_pdl(attn_rows_kernel<D>, dim3(grid), dim3(kRowWarps * 32), smem, s, qr,
                      static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), kr, idx, cnt, mc,
                      dense_all ? 1 : 0, static_cast<__nv_bfloat16*>(out), lse);
}

cudaError_t launch_attn_rows(const QueryRows& qr, const void* k, const void* v, const KvRows& kr, const int32_t* idx,
                             const int32_t* cnt, const MethodConsts& mc, bool dense_all, void* out, float* lse,
                             cudaStream_t s)
{
    return qr.D == 128 ? rows_impl<128>(qr, k, v, kr, idx, cnt, mc, dense_all, out, lse, s)
                       : rows_impl<64>(qr, k, v, kr, idx, cnt, mc, dense_all, out, lse, s);
}

template <int D>
static cudaError_t split_impl(const QueryRows& qr, const void* k, const void* v, const KvRows& kr, const int32_t* idx,
                              const int32_t* cnt, const MethodConsts& mc, bool dense_all, const void* k_draft,
                              const void* v_draft, const uint32_t* tree_mask, void* out, float* lse, void* ws,
                              cudaStream_t s)
{
    const int max_blocks = attn_split_max_blocks(qr.max_ctx, mc.kmax, mc.dense_len, dense_all, mc.window);
    const int nsplit_blocks = attn_split_count(max_blocks);
    const int nsplit_total = nsplit_blocks + (tree_mask ? 1 : 0);
    const size_t smem = (size_t)kSplitWarps * 2 * KvTile<D>::kBytes;
    cudaError_t e = ensure_smem(attn_split_kernel<D>, smem);
    if (e != cudaSuccess) return e;
    const int rows = qr.B * qr.T * qr.Hkv;
    dim3 grid(nsplit_total, rows);
    e = launch_pdl(attn_split_kernel<D>, grid, dim3(kSplitWarps * 32), smem, s, qr,
                   static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), kr, idx, cnt, mc,
                   dense_all ? 1 : 0, nsplit_blocks, static_cast<const __nv_bfloat16*>(k_draft),
                   static_cast<const __nv_bfloat16*>(v_draft), tree_mask, static_cast<float*>(ws));
    if (e != cudaSuccess) return e;
    return launch_pdl(attn_merge_kernel<D>, dim3(rows, qr.Hq / qr.Hkv), dim3(D), 0, s, qr, cnt, mc, dense_all ? 1 : 0,
                      nsplit_blocks, tree_mask ? 1 : 0, static_cast<const float*>(ws),
                      static_cast<__nv_bfloat16*>(out), lse);
}

cudaError_t launch_attn_split(const QueryRows& qr, const void* k, const void* v, const KvRows& kr, const int32_t* idx,
                              const int32_t* cnt, const MethodConsts& mc, bool dense_all, const void* k_draft,
                              const void* v_draft, const uint32_t* tree_mask, void* out, float* lse, void* ws,
                              cudaStream_t s)
{
    return qr.D == 128 ? split_impl<128>(qr, k, v, kr, idx, cnt, mc, dense_all, k_draft, v_draft, tree_mask, out,
                                         lse, ws, s)
                       : split_impl<64>(qr, k, v, kr, idx, cnt, mc, dense_all, k_draft, v_draft, tree_mask, out,
                                        lse, ws, s);
}

}  // namespace iv2

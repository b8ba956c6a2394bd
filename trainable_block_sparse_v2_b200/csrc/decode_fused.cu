// decode_fused.cu -- one decode step of InfLLM v2 (block scoring, top-k, sparse attention) in one kernel.
//
// Same definitions as score.cu and attn.cu ("Tsinghua & ModelBest: MiniCPM4 technical details", "Model
// architecture: InfLLM v2", items 1-3; efficiency evaluation: a decode step reads a constant number of
// blocks plus the slowly growing kernel representations).  A thread-block cluster of CL CTAs owns one
// (sequence, query, KV group) row:
//   1. each CTA bulk-copies its slice of the row's kernel cache (one cp.async.bulk per 128 blocks) into
//      shared memory and scores it on mma.sync (the 16 heads are the MMA rows); it keeps the raw block
//      maxima and per-head (max, sum-exp) partials of its slice;
//   2. after a cluster barrier every CTA merges the CL partials over distributed shared memory into
//      LSE_h, forms the group score S of its blocks and stores it into the leader CTA (rank 0);
//   3. the leader selects (bucket select, select.cuh) and writes idx / cnt;
//   4. every CTA attends to its share of the selected blocks (entries rank, rank + CL, ...), one 64-key
//      block per warp (K/V staged by cp.async into swizzled shared memory, mma.sync, online softmax), and
//      merges its warps;
//   5. CTA r combines every CTA's partial (O, max, sum) of the heads h = r, r + CL, ... over distributed
//      shared memory and writes the output.
// No workspace and no global round trip of partial results; five cluster barriers and no other waits
// (apart from the bounded wait on the CTA's own bulk copy).
#include <cooperative_groups.h>

#include "attn_warp.cuh"
#include "common.cuh"
#include "internal.h"
#include "select.cuh"
#include "tc.cuh"

namespace cg = cooperative_groups;

namespace iv2 {

namespace {

constexpr int kFThreads = 256;                   // 8 warps
constexpr int kFSubBlocks = 128;                 // blocks per scan sub-chunk
constexpr int kFSubRows = 4 * kFSubBlocks + 8;   // kernel rows of a sub-chunk with the halo, whole n-tiles
constexpr int kFMaxBpc = 256;                    // blocks per CTA
constexpr int kFAttnWarps = 5;                   // warps with a K/V buffer in the attention phase

template <int D>
struct FSmem {
    static constexpr int kRows = 0;                                     // kernel rows of a sub-chunk
    static constexpr int kZ = kFSubRows * D * 2;                        // scores [16][kFSubRows]
    static constexpr int kScanEnd = kZ + 16 * kFSubRows * 4;
    static constexpr int kAttnEnd = kFAttnWarps * 2 * kBlock * D * 2;   // K/V tiles per attention warp
    static constexpr int kWarpPart = kFAttnWarps * (16 * D + 32) * 4;   // per-warp (O, m, l) after attention
    static constexpr int kCtaPart = kWarpPart;                          // the CTA's (O[16][D], M[16], L[16])
    static constexpr int kCtaPartEnd = kCtaPart + (16 * D + 32) * 4;
    static constexpr int kRegionA = (kScanEnd > kAttnEnd ? (kScanEnd > kCtaPartEnd ? kScanEnd : kCtaPartEnd)
                                                         : (kAttnEnd > kCtaPartEnd ? kAttnEnd : kCtaPartEnd));
    static constexpr int kBmax = (kRegionA + 127) / 128 * 128;         // [16][kFMaxBpc] raw block maxima
    static constexpr int kS = kBmax + 16 * kFMaxBpc * 4;                // leader: S of every block (4096)
    static constexpr int kBytes = kS + 4096 * 4;
};

// q of one token, G heads as MMA rows, in the permuted head-dimension order of the scan (lane (gq, tq)
// holds d in [8 (4u + tq), +8) of rows gq and gq + 8)
template <int D>
IV2_DEV void fused_q_permuted(const __nv_bfloat16* q_row0, int nrows, uint32_t (&qa)[D / 32][4],
                              uint32_t (&qb)[D / 32][4])
{
    const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int u = 0; u < D / 32; ++u) {
        const int c = 4 * u + tq;
        uint4 va = make_uint4(0, 0, 0, 0), vb = make_uint4(0, 0, 0, 0);
        if (gq < nrows) va = *reinterpret_cast<const uint4*>(q_row0 + (size_t)gq * D + c * 8);
        if (gq + 8 < nrows) vb = *reinterpret_cast<const uint4*>(q_row0 + (size_t)(gq + 8) * D + c * 8);
        qa[u][0] = va.x; qa[u][1] = va.y; qa[u][2] = va.z; qa[u][3] = va.w;
        qb[u][0] = vb.x; qb[u][1] = vb.y; qb[u][2] = vb.z; qb[u][3] = vb.w;
    }
}

__device__ int g_fused_error = 0;

}  // namespace

template <int D, int CL, int E>
__global__ void __launch_bounds__(kFThreads, 1)
decode_fused_kernel(QueryRows qr, const __nv_bfloat16* __restrict__ kern, int nk_cap, MethodConsts mc, int nb_max,
                    const __nv_bfloat16* __restrict__ kc, const __nv_bfloat16* __restrict__ vc, int Lcap,
                    int32_t* __restrict__ idx, int32_t* __restrict__ cnt, __nv_bfloat16* __restrict__ out,
                    float* __restrict__ lse_out)
{
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ __align__(1024) unsigned char smem[];
    __shared__ CtaSelectSmem sel_sm;
    __shared__ float part_m[16], part_s[16], lse_h[16];
    __shared__ uint64_t bar;

    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int row = blockIdx.y;
    const int g = row % qr.Hkv, bt = row / qr.Hkv, t = bt % qr.T, b = bt / qr.T;
    const int G = qr.Hq / qr.Hkv;
    const int n = query_ctx(qr, b, t);
    const int c = (n - 1) / kBlock;
    const bool dense = n <= mc.dense_len;
    const int nkv = min(num_kernels(n), nk_cap);
    const int bpc = (c + CL) / CL;  // blocks per CTA
    const int b0 = rank * bpc, b1 = min(b0 + bpc, c + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
    const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(qr.q) + ((size_t)bt * qr.Hq + g * G) * D;
    int32_t* idx_row = idx + (size_t)row * mc.kmax;
    float* zs = reinterpret_cast<float*>(smem + FSmem<D>::kZ);
    float* bmax = reinterpret_cast<float*>(smem + FSmem<D>::kBmax);
    float* S = reinterpret_cast<float*>(smem + FSmem<D>::kS);

    // ---------------- 1. scan this CTA's slice of the kernel cache ----------------
    if (threadIdx.x < 16) {
        part_m[threadIdx.x] = neg_inf();
        part_s[threadIdx.x] = 0.f;
    }
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        tc::fence_barrier_init();
    }
    __syncthreads();
    if (!dense && b0 <= c) {
        uint32_t qa[D / 32][4], qb[D / 32][4];
        fused_q_permuted<D>(qrow, G, qa, qb);
        const __nv_bfloat16* kbase = kern + ((size_t)b * qr.Hkv + g) * nk_cap * D;
        uint32_t phase = 0;
        for (int sc = b0; sc < b1; sc += kFSubBlocks) {
            const int se = min(sc + kFSubBlocks, b1);
            const int j0 = sc * kKernelsPerBlock - 1, j1 = se * kKernelsPerBlock;  // rows [j0, j1)
            const int lo = max(j0, 0), hi = min(j1, nkv);
            if (hi > lo) {
                if (threadIdx.x == 0) {
                    tc::mbar_arrive_expect_tx(&bar, (uint32_t)(hi - lo) * D * 2);
                    tc::bulk_load(smem + FSmem<D>::kRows + (size_t)(lo - j0) * D * 2, kbase + (size_t)lo * D,
                                  (uint32_t)(hi - lo) * D * 2, &bar);
                }
                if (!tc::mbar_wait(&bar, phase & 1, 1u << 24)) atomicOr(&g_fused_error, 1);
                ++phase;
            }
            const int ntiles = (j1 - j0 + 7) / 8;
            const float scale = mc.scale;
            for (int tile = warp; tile < ntiles; tile += kFThreads / 32) {
                const int jr = j0 + tile * 8 + gq;  // the kernel row this lane supplies
                const bool ok = jr >= lo && jr < hi;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int u = 0; u < D / 32; ++u) {
                    uint4 kv = make_uint4(0, 0, 0, 0);
                    if (ok)
                        kv = *reinterpret_cast<const uint4*>(smem + FSmem<D>::kRows + (size_t)(jr - j0) * D * 2 +
                                                             (4 * u + tq) * 16);
                    const uint32_t a0[4] = {qa[u][0], qb[u][0], qa[u][1], qb[u][1]};
                    mma_bf16_16816(acc, a0, kv.x, kv.y);
                    const uint32_t a1[4] = {qa[u][2], qb[u][2], qa[u][3], qb[u][3]};
                    mma_bf16_16816(acc, a1, kv.z, kv.w);
                }
                const int col0 = tile * 8 + 2 * tq;
                const int ja = j0 + col0, jb = ja + 1;
                const bool va = ja >= lo && ja < hi, vb = jb >= lo && jb < hi;
                zs[gq * kFSubRows + col0] = va ? acc[0] * scale : neg_inf();
                zs[gq * kFSubRows + col0 + 1] = vb ? acc[1] * scale : neg_inf();
                zs[(gq + 8) * kFSubRows + col0] = va ? acc[2] * scale : neg_inf();
                zs[(gq + 8) * kFSubRows + col0 + 1] = vb ? acc[3] * scale : neg_inf();
            }
            __syncthreads();
            // per-head (max, sum-exp) over the owned kernels [4 sc, 4 se) = slots [1, 4 (se - sc)]
            const int nown = kKernelsPerBlock * (se - sc);
            for (int h = warp; h < G; h += kFThreads / 32) {
                float m = neg_inf();
                for (int sl = 1 + lane; sl <= nown; sl += 32) m = fmaxf(m, zs[h * kFSubRows + sl]);
                m = warp_max(m);
                float sum = 0.f;
                if (m != neg_inf())
                    for (int sl = 1 + lane; sl <= nown; sl += 32) sum += exp2_fast((zs[h * kFSubRows + sl] - m) * kLog2e);
                sum = warp_sum(sum);
                if (lane == 0 && m != neg_inf()) {
                    const float pm = part_m[h], M = fmaxf(pm, m);
                    part_s[h] = (pm == neg_inf() ? 0.f : part_s[h] * exp2_fast((pm - M) * kLog2e)) +
                                sum * exp2_fast((m - M) * kLog2e);
                    part_m[h] = M;
                }
            }
            // raw block maxima of the sub-chunk's blocks
            for (int item = threadIdx.x; item < G * (se - sc); item += kFThreads) {
                const int h = item / (se - sc), blk = sc + item % (se - sc);
                int klo, khi;
                block_kernel_range(blk, mc.membership, klo, khi);
                klo = max(klo, 0);
                khi = min(khi, nkv);
                float m = neg_inf();
                for (int j = klo; j < khi; ++j) m = fmaxf(m, zs[h * kFSubRows + (j - j0)]);
                bmax[h * kFMaxBpc + (blk - b0)] = m;
            }
            __syncthreads();
        }
    }
    cluster.sync();  // (1) partials of every CTA visible

    // ---------------- 2. LSE and the group scores of this CTA's blocks ----------------
    if (!dense) {
        if (threadIdx.x < G) {
            const int h = threadIdx.x;
            float M = neg_inf();
            for (int r = 0; r < CL; ++r) M = fmaxf(M, cluster.map_shared_rank(part_m, r)[h]);
            float sum = 0.f;
            if (M != neg_inf())
                for (int r = 0; r < CL; ++r) {
                    const float pm = cluster.map_shared_rank(part_m, r)[h];
                    if (pm != neg_inf()) sum += cluster.map_shared_rank(part_s, r)[h] * exp2_fast((pm - M) * kLog2e);
                }
            lse_h[h] = M == neg_inf() ? neg_inf() : M + logf(sum);
        }
        __syncthreads();
        float* S_leader = cluster.map_shared_rank(S, 0);
        for (int blk = b0 + threadIdx.x; blk < b1; blk += kFThreads) {
            float acc = 0.f;
            bool member = false;
            for (int h = 0; h < G; ++h) {
                const float m = bmax[h * kFMaxBpc + (blk - b0)];
                if (m != neg_inf()) {
                    member = true;
                    acc += exp2_fast((m - lse_h[h]) * kLog2e);
                }
            }
            S_leader[blk] = member ? acc : neg_inf();
        }
    }
    cluster.sync();  // (2) every score in the leader

    // ---------------- 3. selection (leader) ----------------
    if (rank == 0) {
        if (dense) {
            if (threadIdx.x < 32) warp_write_dense_row(c, mc.kmax, idx_row, cnt + row);
        } else {
            cta_select_topk<kFThreads, E>(S, c, mc.init_blocks, mc.local_blocks, mc.topk, mc.kmax, idx_row,
                                          cnt + row, sel_sm);
        }
    }
    cluster.sync();  // (3) idx / cnt of the row written (release/acquire at cluster scope)

    // ---------------- 4. attention over this CTA's share of the blocks ----------------
    const int count = dense ? c + 1 : min(cnt[row], mc.kmax);
    WarpAttnState<D> st;
    st.init();
    bool worked = false;
    if (warp < kFAttnWarps) {
        uint32_t qf[D / 16][4];
        load_q_rows<D>(qrow, G, qf);
        unsigned char* ks_tile = smem + warp * 2 * KvTile<D>::kBytes;
        unsigned char* vs_tile = ks_tile + KvTile<D>::kBytes;
        const size_t rs = (size_t)qr.Hkv * D;
        const __nv_bfloat16* kb = kc + ((size_t)b * Lcap * qr.Hkv + g) * D;
        const __nv_bfloat16* vb = vc + ((size_t)b * Lcap * qr.Hkv + g) * D;
        const float sl2 = mc.scale * kLog2e;
        for (int i = warp;; i += kFAttnWarps) {
            const int e = rank + CL * i;
            if (e >= count) break;
            const int blk = dense ? e : idx_row[e];
            if (blk < 0 || blk * kBlock >= n) continue;
            const int nvalid = min(kBlock, n - blk * kBlock);
            warp_load_tile<D>(ks_tile, kb + (size_t)blk * kBlock * rs, rs, nvalid);
            warp_load_tile<D>(vs_tile, vb + (size_t)blk * kBlock * rs, rs, nvalid);
            cp_async_commit();
            cp_async_wait<0>();
            __syncwarp();
            float acc[8][4];
            tile_qk<D>(qf, ks_tile, acc);
            scale_mask(acc, sl2, prefix_mask64(nvalid));
            tile_softmax_pv<D>(st, acc, vs_tile);
            __syncwarp();
            worked = true;
        }
        finalize_rows<D>(st);
    }
    __syncthreads();  // K/V tiles are dead: the region holds the per-warp and CTA partials from here on
    float* wo = reinterpret_cast<float*>(smem);                        // [kFAttnWarps][16][D]
    float* wm = wo + kFAttnWarps * 16 * D;                             // [kFAttnWarps][16]
    float* wl = wm + kFAttnWarps * 16;                                 // [kFAttnWarps][16]
    float* co = reinterpret_cast<float*>(smem + FSmem<D>::kCtaPart);  // [16][D]
    float* cm = co + 16 * D;                                           // [16]
    float* cl = cm + 16;                                               // [16]
    if (warp < kFAttnWarps) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int r = gq + 8 * i;
#pragma unroll
            for (int nd = 0; nd < D / 8; ++nd) {
                wo[(warp * 16 + r) * D + nd * 8 + 2 * tq] = st.o[nd][2 * i];
                wo[(warp * 16 + r) * D + nd * 8 + 2 * tq + 1] = st.o[nd][2 * i + 1];
            }
            if (tq == 0) {
                wm[warp * 16 + r] = worked ? st.m[i] : neg_inf();
                wl[warp * 16 + r] = worked ? st.l[i] : 0.f;
            }
        }
    }
    __syncthreads();
    for (int item = threadIdx.x; item < 16 * D; item += kFThreads) {
        const int r = item / D, d = item % D;
        float M = neg_inf();
#pragma unroll
        for (int w = 0; w < kFAttnWarps; ++w) M = fmaxf(M, wm[w * 16 + r]);
        float O = 0.f, L = 0.f;
        if (M != neg_inf()) {
#pragma unroll
            for (int w = 0; w < kFAttnWarps; ++w) {
                const float f = exp2_fast(wm[w * 16 + r] - M);
                O += wo[(w * 16 + r) * D + d] * f;
                L += wl[w * 16 + r] * f;
            }
        }
        co[r * D + d] = O;
        if (d == 0) {
            cm[r] = M;
            cl[r] = L;
        }
    }
    cluster.sync();  // (4) every CTA's partial visible

    // ---------------- 5. combine the CTAs' partials; CTA `rank` writes heads rank, rank + CL, ... ----------------
    for (int h = rank; h < G; h += CL) {
        for (int d = threadIdx.x; d < D; d += kFThreads) {
            float M = neg_inf();
            for (int r = 0; r < CL; ++r) M = fmaxf(M, cluster.map_shared_rank(cm, r)[h]);
            float O = 0.f, L = 0.f;
            if (M != neg_inf())
                for (int r = 0; r < CL; ++r) {
                    const float mr = cluster.map_shared_rank(cm, r)[h];
                    if (mr == neg_inf()) continue;
                    const float f = exp2_fast(mr - M);
                    O += cluster.map_shared_rank(co, r)[h * D + d] * f;
                    L += cluster.map_shared_rank(cl, r)[h] * f;
                }
            out[((size_t)bt * qr.Hq + g * G + h) * D + d] = __float2bfloat16_rn(L > 0.f ? O / L : 0.f);
            if (lse_out && d == 0)
                lse_out[(size_t)bt * qr.Hq + g * G + h] = L > 0.f ? (M + __log2f(L)) * kLn2 : neg_inf();
        }
    }
    cluster.sync();  // (5) no CTA leaves while its partial may still be read
}

// ---------------------------------------------------------------- host
template <int D, int CL, int E>
static cudaError_t fused_launch(const QueryRows& qr, const void* kern, int nk_cap, const MethodConsts& mc, int nb_max,
                                const void* k, const void* v, int Lcap, int32_t* idx, int32_t* cnt, void* out,
                                float* lse, cudaStream_t s)
{
    auto kfn = decode_fused_kernel<D, CL, E>;
    cudaError_t e = ensure_smem(kfn, FSmem<D>::kBytes);
    if (e != cudaSuccess) return e;
    if (CL > 8) {
        e = cudaFuncSetAttribute(kfn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    const int rows = qr.B * qr.T * qr.Hkv;
    return launch_pdl_cluster(kfn, dim3(CL, rows), dim3(kFThreads), CL, FSmem<D>::kBytes, s, qr,
                              static_cast<const __nv_bfloat16*>(kern), nk_cap, mc, nb_max,
                              static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), Lcap, idx,
                              cnt, static_cast<__nv_bfloat16*>(out), lse);
}

// largest cluster size the device schedules for this kernel (16 when the GPU allows it, else 8)
template <int D, int E>
static int fused_cluster_size()
{
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 8;
    if (cached[dev]) return cached[dev];
    int cl = 8;
    auto kfn = decode_fused_kernel<D, 16, E>;
    if (ensure_smem(kfn, FSmem<D>::kBytes) == cudaSuccess &&
        cudaFuncSetAttribute(kfn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(16, 1);
        cfg.blockDim = dim3(kFThreads);
        cfg.dynamicSmemBytes = FSmem<D>::kBytes;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 16;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int nclusters = 0;
        if (cudaOccupancyMaxActiveClusters(&nclusters, kfn, &cfg) == cudaSuccess && nclusters >= 1) cl = 16;
    }
    (void)cudaGetLastError();
    cached[dev] = cl;
    return cl;
}

template <int D, int E>
static cudaError_t fused_dispatch_cl(const QueryRows& qr, const void* kern, int nk_cap, const MethodConsts& mc,
                                     int nb_max, const void* k, const void* v, int Lcap, int32_t* idx, int32_t* cnt,
                                     void* out, float* lse, cudaStream_t s)
{
    const int cl = (nb_max <= 8 * kFMaxBpc) ? fused_cluster_size<D, E>() : 16;
    if (cl == 16) return fused_launch<D, 16, E>(qr, kern, nk_cap, mc, nb_max, k, v, Lcap, idx, cnt, out, lse, s);
    return fused_launch<D, 8, E>(qr, kern, nk_cap, mc, nb_max, k, v, Lcap, idx, cnt, out, lse, s);
}

bool decode_fused_supported(const QueryRows& qr, const MethodConsts& mc)
{
    const int nb_max = (qr.max_ctx - 1) / kBlock + 1;
    return nb_max <= 16 * kFMaxBpc && qr.Hq / qr.Hkv <= 16 && (qr.D == 64 || qr.D == 128) && mc.kmax <= 4096;
}

cudaError_t launch_decode_fused(const QueryRows& qr, const void* kern, int nk_cap, const MethodConsts& mc,
                                const void* k, const void* v, int Lcap, int32_t* idx, int32_t* cnt, void* out,
                                float* lse, cudaStream_t s)
{
    const int nb_max = (qr.max_ctx - 1) / kBlock + 1;
    if (!decode_fused_supported(qr, mc)) return cudaErrorNotSupported;
    // the leader's top-k keeps ceil(nb_max / 256) blocks per thread
    if (qr.D == 128) {
        if (nb_max <= 1024) return fused_dispatch_cl<128, 4>(qr, kern, nk_cap, mc, nb_max, k, v, Lcap, idx, cnt, out, lse, s);
        if (nb_max <= 2048) return fused_dispatch_cl<128, 8>(qr, kern, nk_cap, mc, nb_max, k, v, Lcap, idx, cnt, out, lse, s);
        return fused_dispatch_cl<128, 16>(qr, kern, nk_cap, mc, nb_max, k, v, Lcap, idx, cnt, out, lse, s);
    }
    if (nb_max <= 1024) return fused_dispatch_cl<64, 4>(qr, kern, nk_cap, mc, nb_max, k, v, Lcap, idx, cnt, out, lse, s);
    if (nb_max <= 2048) return fused_dispatch_cl<64, 8>(qr, kern, nk_cap, mc, nb_max, k, v, Lcap, idx, cnt, out, lse, s);
    return fused_dispatch_cl<64, 16>(qr, kern, nk_cap, mc, nb_max, k, v, Lcap, idx, cnt, out, lse, s);
}

int fused_error_flag_read_and_clear()
{
    int h = 0;
    if (cudaMemcpyFromSymbol(&h, g_fused_error, sizeof(int)) != cudaSuccess) return -1;
    if (h) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_fused_error, &zero, sizeof(int));
    }
    return h;
}

}  // namespace iv2

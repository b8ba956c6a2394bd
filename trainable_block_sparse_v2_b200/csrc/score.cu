// score.cu -- block scoring and top-k selection (step 2 of InfLLM v2).
//
// For query (b, t), KV group g and head h of the group (MiniCPM4 technical details, "Model architecture:
// InfLLM v2": item 1 max over a block's semantic kernels, item 2 one block set per GQA group, item 3
// LogSumExp normalisation and top-k):
//   z_h(j)   = scale * q_h . kern_j        for the visible kernels j < nk(n)
//   LSE_h    = log sum_j exp z_h(j)         (exact)
//   S_g(blk) = sum_h exp(max_{j in blk} z_h(j) - LSE_h)
// then top-k over S_g with the forced blocks (select.cuh).
//
// Two layouts of the same computation:
//  * few query rows (decode, tree verification): the kernel cache is the HBM stream.  Each CTA scans a
//    chunk of 32 blocks (128 kernels) of one row with mma.sync m16n8k16 (the G heads of the group are the
//    16 MMA rows), writing per-head partial (max, sum-exp) and raw block maxima; a second kernel merges
//    the partials into LSE_h, forms S_g and selects, one CTA per row.  Kernel rows are loaded straight
//    into MMA fragments with 16-byte loads: the head dimension is visited in a permuted order that is the
//    same for q and the kernels, so a dot product is unchanged.
//  * many query rows (prefill): a CTA takes a tile of consecutive tokens of one group (each warp: 16 MMA
//    rows = 16/G tokens x G heads) and streams 64-kernel tiles through shared memory (cp.async, swizzled
//    for ldmatrix).  Pass 1 accumulates LSE_h online; pass 2 recomputes the scores, max-pools them into
//    blocks, normalises, sums over the group and keeps S in shared memory; each warp then selects for
//    its tokens.  No S or LSE ever goes to global memory.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace cg = cooperative_groups;

namespace iv2 {

// =====================================================================================================
// few rows: split-kernel scan
// =====================================================================================================
constexpr int kChunkBlocks = 32;
constexpr int kChunkKernels = kChunkBlocks * kKernelsPerBlock;   // 128 kernels owned per CTA
constexpr int kChunkSlots = kChunkKernels + 8;                  // + halo kernel, rounded to n-tiles
constexpr int kScanThreads = 128;

struct ScoreWs {
    float* pmax;   // [rows, nchunk, 16]
    float* psum;   // [rows, nchunk, 16]
    float* bmax;   // [rows, 16, nb_max]
};

__host__ __device__ inline int score_nchunk(int nb_max) { return (nb_max + kChunkBlocks - 1) / kChunkBlocks; }

// q fragments in the permuted head-dimension order: for u in [0, D/32), lane (gq, tq) holds the 8 values
// d in [8 (4u + tq), +8) of rows gq and gq + 8.
template <int D>
IV2_DEV void load_q_permuted(const __nv_bfloat16* q_row0, int nrows, uint32_t (&qa)[D / 32][4],
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

template <int D>
__global__ void __launch_bounds__(kScanThreads) score_scan_kernel(QueryRows qr, const __nv_bfloat16* __restrict__ kern,
                                                                  int nk_cap, MethodConsts mc, int nb_max, ScoreWs ws)
{
    pdl_launch_dependents();
    pdl_wait();
    __shared__ float zs[16][kChunkSlots];
    const int row = blockIdx.y;  // (b, t, g); the workspace is indexed by it
    const int g = row % qr.Hkv, t = (row / qr.Hkv) % qr.T, b = row / qr.Hkv / qr.T;
    if (t >= q_len(qr, b)) return;  // past this sequence's queries (packed batch)
    const long bt = q_row(qr, b, t);
    const int G = qr.Hq / qr.Hkv;
    const int n = query_ctx(qr, b, t);
    if (n <= mc.dense_len) return;
    const int c = (n - 1) / kBlock;
    const int cb0 = blockIdx.x * kChunkBlocks;
    if (cb0 > c) return;
    const int nkv = min(num_kernels(n), nk_cap);
    const int j0 = cb0 * kKernelsPerBlock - 1;  // kernel of slot 0

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
    uint32_t qa[D / 32][4], qb[D / 32][4];
    load_q_permuted<D>(static_cast<const __nv_bfloat16*>(qr.q) + ((size_t)bt * qr.Hq + g * G) * D, G, qa, qb);
    const __nv_bfloat16* kbase = kern + ((size_t)b * qr.Hkv + g) * nk_cap * D;
    const float scale = mc.scale;

    // tiles warp, warp + 4, ...: issue every kernel-row load of the warp first, then the MMAs
    constexpr int kTiles = kChunkSlots / 8;                                            // 17
    constexpr int kPerWarp = (kTiles + kScanThreads / 32 - 1) / (kScanThreads / 32);  // 5
    uint4 kv[kPerWarp][D / 32];
#pragma unroll
    for (int i = 0; i < kPerWarp; ++i) {
        const int tile = warp + i * (kScanThreads / 32);
        const int jr = j0 + tile * 8 + gq;  // the kernel row this lane loads
        const bool ok = tile < kTiles && jr >= 0 && jr < nkv;
#pragma unroll
        for (int u = 0; u < D / 32; ++u)
            kv[i][u] = ok ? ld_nc_v4(kbase + (size_t)jr * D + (4 * u + tq) * 8) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < kPerWarp; ++i) {
        const int tile = warp + i * (kScanThreads / 32);
        if (tile >= kTiles) break;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int u = 0; u < D / 32; ++u) {
            const uint32_t a0[4] = {qa[u][0], qb[u][0], qa[u][1], qb[u][1]};
            mma_bf16_16816(acc, a0, kv[i][u].x, kv[i][u].y);
            const uint32_t a1[4] = {qa[u][2], qb[u][2], qa[u][3], qb[u][3]};
            mma_bf16_16816(acc, a1, kv[i][u].z, kv[i][u].w);
        }
        const int col0 = tile * 8 + 2 * tq;
        const int ja = j0 + col0, jb = ja + 1;
        const bool va = ja >= 0 && ja < nkv, vb = jb >= 0 && jb < nkv;
        zs[gq][col0] = va ? acc[0] * scale : neg_inf();
        zs[gq][col0 + 1] = vb ? acc[1] * scale : neg_inf();
        zs[gq + 8][col0] = va ? acc[2] * scale : neg_inf();
        zs[gq + 8][col0 + 1] = vb ? acc[3] * scale : neg_inf();
    }
    __syncthreads();

    const int nchunk = score_nchunk(nb_max);
    // per-head partial LSE over the owned kernels (slots 1 .. kChunkKernels)
    for (int h = warp; h < G; h += kScanThreads / 32) {
        float m = neg_inf();
        for (int s = 1 + lane; s <= kChunkKernels; s += 32) m = fmaxf(m, zs[h][s]);
        m = warp_max(m);
        float sum = 0.f;
        if (m != neg_inf())
            for (int s = 1 + lane; s <= kChunkKernels; s += 32) sum += exp2_fast((zs[h][s] - m) * kLog2e);
        sum = warp_sum(sum);
        if (lane == 0) {
            ws.pmax[((size_t)row * nchunk + blockIdx.x) * 16 + h] = m;
            ws.psum[((size_t)row * nchunk + blockIdx.x) * 16 + h] = sum;
        }
    }
    // raw block maxima, head-major: bmax[row][h][blk] (consecutive threads write consecutive blocks)
    const int nblk = min(kChunkBlocks, c + 1 - cb0);
    for (int item = threadIdx.x; item < G * kChunkBlocks; item += kScanThreads) {
        const int h = item / kChunkBlocks, bl = item % kChunkBlocks, blk = cb0 + bl;
        if (bl >= nblk) continue;
        int lo, hi;
        block_kernel_range(blk, mc.membership, lo, hi);
        lo = max(lo, 0);
        hi = min(hi, nkv);
        float m = neg_inf();
        for (int j = lo; j < hi; ++j) m = fmaxf(m, zs[h][j - j0]);
        ws.bmax[((size_t)row * 16 + h) * nb_max + blk] = m;
    }
}

// The select of one row runs on a cluster of kSelCluster CTAs: every CTA merges the chunk partials into
// LSE_h, forms S for 1/kSelCluster of the blocks (its block maxima are a contiguous head-major slice) and
// stores them into the leader CTA's shared memory over distributed shared memory; after one cluster
// barrier the leader (rank 0) selects.  Spreading the block maxima over 8 SMs is what makes this fast:
// a single SM pulls the 128 KB of a 128K-context row far too slowly.
constexpr int kSelCluster = 8;
constexpr int kSelThreads = 512;  // the leader's top-k: up to 8 blocks per thread -> nb_max <= 4096

template <int E>
__global__ void __launch_bounds__(kSelThreads) score_select_kernel(QueryRows qr, MethodConsts mc, int nb_max,
                                                                   ScoreWs ws, int32_t* __restrict__ idx,
                                                                   int32_t* __restrict__ cnt)
{
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ float S[];  // nb_max; the leader's copy receives every CTA's scores
    __shared__ float lse[16];
    __shared__ CtaSelectSmem sel_sm;
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int row = blockIdx.y;  // (b, t, g): the workspace row
    const int t = (row / qr.Hkv) % qr.T, b = row / qr.Hkv / qr.T;
    if (t >= q_len(qr, b)) return;  // past this sequence's queries: uniform over the cluster
    const long orow = q_row(qr, b, t) * qr.Hkv + row % qr.Hkv;  // row of idx / cnt
    const int G = qr.Hq / qr.Hkv;
    const int n = query_ctx(qr, b, t);
    const int c = (n - 1) / kBlock;
    int32_t* idx_row = idx + (size_t)orow * mc.kmax;
    if (n <= mc.dense_len) {  // uniform over the cluster: nobody touches distributed shared memory
        if (rank == 0 && threadIdx.x < 32) warp_write_dense_row(c, mc.kmax, idx_row, cnt + orow);
        return;
    }
    const int nchunk = score_nchunk(nb_max);
    const int nch_row = c / kChunkBlocks + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's blocks and their raw maxima (loaded first: the load overlaps the LSE merge)
    const int per = (c + kSelCluster) / kSelCluster;  // ceil((c + 1) / kSelCluster) <= kSelThreads
    const int blk = rank * per + (int)threadIdx.x;
    const bool mine = (int)threadIdx.x < per && blk <= c;
    float mb[16];
#pragma unroll
    for (int h = 0; h < 16; ++h)
        mb[h] = (mine && h < G) ? ws.bmax[((size_t)row * 16 + h) * nb_max + blk] : neg_inf();
    if (warp < G) {
        // LSE_h from the chunk partials: both loads in flight together
        const int h = warp;
        constexpr int kMaxChunkPerLane = 4;  // nb_max <= 4096 blocks -> <= 128 chunks
        float pm[kMaxChunkPerLane], ps[kMaxChunkPerLane];
#pragma unroll
        for (int u = 0; u < kMaxChunkPerLane; ++u) {
            const int i = lane + 32 * u;
            const bool ok = i < nch_row;
            pm[u] = ok ? ws.pmax[((size_t)row * nchunk + i) * 16 + h] : neg_inf();
            ps[u] = ok ? ws.psum[((size_t)row * nchunk + i) * 16 + h] : 0.f;
        }
        float m = neg_inf();
#pragma unroll
        for (int u = 0; u < kMaxChunkPerLane; ++u) m = fmaxf(m, pm[u]);
        m = warp_max(m);
        float ssum = 0.f;
        if (m != neg_inf())
#pragma unroll
            for (int u = 0; u < kMaxChunkPerLane; ++u)
                if (pm[u] != neg_inf()) ssum += ps[u] * exp2_fast((pm[u] - m) * kLog2e);
        ssum = warp_sum(ssum);
        if (lane == 0) lse[h] = (m == neg_inf()) ? neg_inf() : m + logf(ssum);
    }
    __syncthreads();
    if (mine) {
        // every head of the group sees the same kernels: a block without a visible kernel is -inf for all
        float acc = 0.f;
#pragma unroll
        for (int h = 0; h < 16; ++h)
            if (h < G && mb[h] != neg_inf()) acc += exp2_fast((mb[h] - lse[h]) * kLog2e);
        float* S_leader = cluster.map_shared_rank(S, 0);
        S_leader[blk] = mb[0] != neg_inf() ? acc : neg_inf();
    }
    cluster.sync();  // release/acquire: the leader sees every score
    if (rank != 0) return;
    cta_select_topk<kSelThreads, E>(S, c, mc.init_blocks, mc.local_blocks, mc.topk, mc.kmax, idx_row, cnt + orow,
                                    sel_sm);
}

// =====================================================================================================
// many rows: token tiles
// =====================================================================================================
constexpr int kPfWarps = 8;
constexpr int kPfThreads = kPfWarps * 32;
constexpr int kKT = 64;  // kernels per shared-memory tile

template <int D>
struct PfSmem {
    static constexpr int kTileBytes = kKT * D * 2;
};

// swizzled tile: row r (kernel), 16-byte chunk ch -> byte offset r*D*2 + ((ch ^ (r & 7)) * 16)
template <int D>
IV2_DEV uint32_t swz(int r, int ch)
{
    return (uint32_t)(r * D * 2 + ((ch ^ (r & 7)) << 4));
}

template <int D>
IV2_DEV void pf_load_tile(unsigned char* dst, const __nv_bfloat16* kbase, int jt0, int nk_lim)
{
    constexpr int CH = D / 8;
    for (int i = threadIdx.x; i < kKT * CH; i += kPfThreads) {
        const int r = i / CH, ch = i % CH;
        const int j = jt0 + r;
        const bool ok = j < nk_lim;
        cp_async_16_zfill(dst + swz<D>(r, ch), kbase + (size_t)(ok ? j : 0) * D + ch * 8, ok ? 16 : 0);
    }
}

// scores of the warp's 16 rows against the 64 kernels of a tile: acc[nt][4] for n-tiles nt = 0..7
template <int D>
IV2_DEV void pf_tile_scores(const uint32_t (&qf)[D / 16][4], const unsigned char* tile, float (&acc)[8][4])
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ks += 2) {
            // matrices: (chunk 2ks, 2ks+1, 2ks+2, 2ks+3) x rows nt*8 .. +7
            const int r = nt * 8 + (lane & 7);
            const int ch = 2 * ks + (lane >> 3);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(b0, b1, b2, b3, tile + swz<D>(r, ch));
            mma_bf16_16816(acc[nt], qf[ks], b0, b1);
            mma_bf16_16816(acc[nt], qf[ks + 1], b2, b3);
        }
    }
}

template <int D, int G>
__global__ void __launch_bounds__(kPfThreads) score_prefill_kernel(QueryRows qr, const __nv_bfloat16* __restrict__ kern,
                                                                   int nk_cap, MethodConsts mc, int nb_max,
                                                                   int32_t* __restrict__ idx, int32_t* __restrict__ cnt)
{
    pdl_launch_dependents();
    pdl_wait();
    constexpr int TW = 16 / G;               // tokens per warp
    constexpr int TPC = TW * kPfWarps;       // tokens per CTA
    constexpr int ZW = 72;                   // z row: column 7 = previous tile's last kernel, 8.. = this tile
    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char* tiles = smem;                                              // 2 x tile
    float* zw = reinterpret_cast<float*>(smem + 2 * PfSmem<D>::kTileBytes);  // [warps][16][ZW]
    float* Ssm = zw + kPfWarps * 16 * ZW;                                     // [TPC][nb_max]
    __shared__ float lsew[kPfWarps][16];
    __shared__ int n_max_sh;

    const int g = blockIdx.y % qr.Hkv, b = blockIdx.y / qr.Hkv;
    const int t0 = blockIdx.x * TPC;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
    const int T = q_len(qr, b);  // this sequence's queries (qr.T unless the batch is packed)
    if (t0 >= T) return;         // uniform over the CTA, before any barrier

    if (threadIdx.x == 0) n_max_sh = 0;
    __syncthreads();
    if (threadIdx.x < TPC && t0 + threadIdx.x < T)
        atomicMax(&n_max_sh, query_ctx(qr, b, t0 + threadIdx.x));
    __syncthreads();
    const int n_max = n_max_sh;
    const bool any_sparse = n_max > mc.dense_len;
    const int nk_tile_lim = min(num_kernels(n_max), nk_cap);

    // rows of this warp: r = tt * G + hh  (token tw0 + tt, head g*G + hh)
    const int tw0 = t0 + warp * TW;
    int nkv_row[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int tk = tw0 + (gq + 8 * i) / G;
        nkv_row[i] = tk < T ? min(num_kernels(query_ctx(qr, b, tk)), nk_cap) : 0;
    }

    uint32_t qf[D / 16][4];
    const __nv_bfloat16* qbase = static_cast<const __nv_bfloat16*>(qr.q);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = gq + 8 * (i & 1);
            const int dcol = ks * 16 + 2 * tq + 8 * (i >> 1);
            const int tt = r / G, hh = r % G, tk = tw0 + tt;
            qf[ks][i] = 0u;
            if (any_sparse && tk < T)
                qf[ks][i] = *reinterpret_cast<const uint32_t*>(
                    qbase + ((size_t)q_row(qr, b, tk) * qr.Hq + g * G + hh) * D + dcol);
        }
    }

    const __nv_bfloat16* kbase = kern + ((size_t)b * qr.Hkv + g) * nk_cap * D;
    // every block up to the last token's own block gets a score (16 blocks end in each tile)
    const int ntiles = any_sparse ? max((nk_tile_lim + kKT - 1) / kKT, (n_max - 1) / kBlock / 16 + 1) : 0;
    const float sl2 = mc.scale * kLog2e;  // scores kept in log2 units

    // ---------------- pass 1: LSE of every row (online over the tiles) -----------------
    float rm[2] = {neg_inf(), neg_inf()}, rs[2] = {0.f, 0.f};
    if (ntiles > 0) {
        pf_load_tile<D>(tiles, kbase, 0, nk_tile_lim);
        cp_async_commit();
    }
    for (int it = 0; it < ntiles; ++it) {
        if (it + 1 < ntiles) {
            pf_load_tile<D>(tiles + ((it + 1) & 1) * PfSmem<D>::kTileBytes, kbase, (it + 1) * kKT, nk_tile_lim);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        float acc[8][4];
        pf_tile_scores<D>(qf, tiles + (it & 1) * PfSmem<D>::kTileBytes, acc);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float m = rm[i];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int j = it * kKT + nt * 8 + 2 * tq + e;
                    if (j < nkv_row[i]) m = fmaxf(m, acc[nt][2 * i + e] * sl2);
                }
            if (m != neg_inf()) {
                float sum = rs[i] * exp2_fast(rm[i] - m);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int j = it * kKT + nt * 8 + 2 * tq + e;
                        if (j < nkv_row[i]) sum += exp2_fast(acc[nt][2 * i + e] * sl2 - m);
                    }
                rs[i] = sum;
                rm[i] = m;
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        float m = rm[i];
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        float sum = (m == neg_inf()) ? 0.f : rs[i] * exp2_fast(rm[i] - m);
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        if (tq == 0) lsew[warp][gq + 8 * i] = (m == neg_inf()) ? neg_inf() : m + __log2f(sum);
    }

    // ---------------- pass 2: block maxima -> normalised -> summed over the group -----------------
    float* z = zw + warp * 16 * ZW;
    float* Sw = Ssm + (size_t)(warp * TW) * nb_max;
    if (lane < 16) z[lane * ZW + 7] = neg_inf();
    __syncwarp();
    if (ntiles > 0) {
        pf_load_tile<D>(tiles, kbase, 0, nk_tile_lim);
        cp_async_commit();
    }
    for (int it = 0; it < ntiles; ++it) {
        if (it + 1 < ntiles) {
            pf_load_tile<D>(tiles + ((it + 1) & 1) * PfSmem<D>::kTileBytes, kbase, (it + 1) * kKT, nk_tile_lim);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        float acc[8][4];
        pf_tile_scores<D>(qf, tiles + (it & 1) * PfSmem<D>::kTileBytes, acc);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int col = nt * 8 + 2 * tq + e;
                    const int j = it * kKT + col;
                    z[(gq + 8 * i) * ZW + 8 + col] = j < nkv_row[i] ? acc[nt][2 * i + e] * sl2 : neg_inf();
                }
        __syncwarp();
        // the 16 blocks whose kernels end in this tile, for each of the warp's tokens
        for (int item = lane; item < TW * 16; item += 32) {
            const int tt = item / 16, blk = it * 16 + item % 16;
            const int tk = tw0 + tt;
            if (tk >= T) continue;
            const int n = query_ctx(qr, b, tk);
            if (blk > (n - 1) / kBlock || blk >= nb_max) continue;
            const int nkv = min(num_kernels(n), nk_cap);
            int lo, hi;
            block_kernel_range(blk, mc.membership, lo, hi);
            lo = max(lo, 0);
            hi = min(hi, nkv);
            float sacc = 0.f;
            if (lo < hi) {
                for (int hh = 0; hh < G; ++hh) {
                    const int r = tt * G + hh;
                    float m = neg_inf();
                    for (int j = lo; j < hi; ++j) m = fmaxf(m, z[r * ZW + 8 + j - it * kKT]);
                    sacc += exp2_fast(m - lsew[warp][r]);
                }
            }
            Sw[(size_t)tt * nb_max + blk] = lo < hi ? sacc : neg_inf();
        }
        __syncwarp();
        if (lane < 16) z[lane * ZW + 7] = z[lane * ZW + 8 + kKT - 1];
        __syncthreads();
    }
    __syncwarp();

    // ---------------- selection, one warp per token -----------------
    for (int tt = 0; tt < TW; ++tt) {
        const int tk = tw0 + tt;
        if (tk >= T) break;
        const int n = query_ctx(qr, b, tk);
        const int c = (n - 1) / kBlock;
        const size_t row = (size_t)q_row(qr, b, tk) * qr.Hkv + g;
        if (n <= mc.dense_len)
            warp_write_dense_row(c, mc.kmax, idx + row * mc.kmax, cnt + row);
        else
            warp_select_topk(Sw + (size_t)tt * nb_max, c, mc.init_blocks, mc.local_blocks, mc.topk, mc.kmax,
                             idx + row * mc.kmax, cnt + row);
    }
}

// =====================================================================================================
// host side
// =====================================================================================================
static int nb_of(int max_ctx) { return (max_ctx - 1) / kBlock + 1; }

size_t score_ws_bytes(int rows, int max_ctx)
{
    const int nb_max = nb_of(max_ctx);
    const size_t nchunk = (size_t)(nb_max + kChunkBlocks - 1) / kChunkBlocks;
    auto al = [](size_t x) { return (x + 255) / 256 * 256; };
    return al((size_t)rows * nchunk * 16 * 4) * 2 + al((size_t)rows * 16 * nb_max * 4);
}

static size_t prefill_score_smem(int G, int D, int nb_max)
{
    const int TPC = (16 / G) * kPfWarps;
    return 2 * (size_t)kKT * D * 2 + (size_t)kPfWarps * 16 * 72 * 4 + (size_t)TPC * nb_max * 4;
}

static constexpr size_t kPfSmemLimit = 220 * 1024;

// token tiles unless there are too few queries to fill the GPU or the tile's scores exceed shared memory
bool score_uses_scan_path(int B, int T, int G, int D, int max_ctx)
{
    return (long)B * T <= 64 || prefill_score_smem(G, D, nb_of(max_ctx)) > kPfSmemLimit;
}

template <int D, int G>
static cudaError_t launch_prefill_score(const QueryRows& qr, const __nv_bfloat16* kern, int nk_cap,
                                        const MethodConsts& mc, int nb_max, int32_t* idx, int32_t* cnt, cudaStream_t s)
{
    constexpr int TPC = (16 / G) * kPfWarps;
    const size_t smem = prefill_score_smem(G, D, nb_max);
    cudaError_t e = ensure_smem(score_prefill_kernel<D, G>, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((qr.T + TPC - 1) / TPC, qr.B * qr.Hkv);
    return launch_pdl(score_prefill_kernel<D, G>, grid, dim3(kPfThreads), smem, s, qr, kern, nk_cap, mc, nb_max, idx,
                      cnt);
}

template <int D>
static cudaError_t launch_prefill_score_g(const QueryRows& qr, const __nv_bfloat16* kern, int nk_cap,
                                          const MethodConsts& mc, int nb_max, int32_t* idx, int32_t* cnt,
                                          cudaStream_t s)
{
    switch (qr.Hq / qr.Hkv) {
    case 1: return launch_prefill_score<D, 1>(qr, kern, nk_cap, mc, nb_max, idx, cnt, s);
    case 2: return launch_prefill_score<D, 2>(qr, kern, nk_cap, mc, nb_max, idx, cnt, s);
    case 4: return launch_prefill_score<D, 4>(qr, kern, nk_cap, mc, nb_max, idx, cnt, s);
    case 8: return launch_prefill_score<D, 8>(qr, kern, nk_cap, mc, nb_max, idx, cnt, s);
    default: return launch_prefill_score<D, 16>(qr, kern, nk_cap, mc, nb_max, idx, cnt, s);
    }
}

cudaError_t launch_score_topk(const QueryRows& qr, const void* kern_v, int nk_cap, const MethodConsts& mc,
                              int32_t* idx, int32_t* cnt, void* ws, cudaStream_t s)
{
    const __nv_bfloat16* kern = static_cast<const __nv_bfloat16*>(kern_v);
    const int nb_max = nb_of(qr.max_ctx);
    if (!score_uses_scan_path(qr.B, qr.T, qr.Hq / qr.Hkv, qr.D, qr.max_ctx)) {
        if (score_tc_supported(qr, nb_max)) return launch_score_tc(qr, kern, nk_cap, mc, nb_max, idx, cnt, s);
        return qr.D == 128 ? launch_prefill_score_g<128>(qr, kern, nk_cap, mc, nb_max, idx, cnt, s)
                           : launch_prefill_score_g<64>(qr, kern, nk_cap, mc, nb_max, idx, cnt, s);
    }
    const int rows = qr.B * qr.T * qr.Hkv;
    const int nchunk = score_nchunk(nb_max);
    auto al = [](size_t x) { return (x + 255) / 256 * 256; };
    char* w = static_cast<char*>(ws);
    ScoreWs sw;
    sw.pmax = reinterpret_cast<float*>(w);
    sw.psum = reinterpret_cast<float*>(w + al((size_t)rows * nchunk * 16 * 4));
    sw.bmax = reinterpret_cast<float*>(w + 2 * al((size_t)rows * nchunk * 16 * 4));
    dim3 g1(nchunk, rows);
    cudaError_t e = qr.D == 128
                        ? launch_pdl(score_scan_kernel<128>, g1, dim3(kScanThreads), 0, s, qr, kern, nk_cap, mc, nb_max, sw)
                        : launch_pdl(score_scan_kernel<64>, g1, dim3(kScanThreads), 0, s, qr, kern, nk_cap, mc, nb_max, sw);
    if (e != cudaSuccess) return e;
    const size_t smem = (size_t)nb_max * 4;
    const int E = (nb_max + kSelThreads - 1) / kSelThreads;
    const dim3 g2(kSelCluster, rows), b2(kSelThreads);
    switch (E) {
    case 1: return launch_pdl_cluster(score_select_kernel<1>, g2, b2, kSelCluster, smem, s, qr, mc, nb_max, sw, idx, cnt);
    case 2: return launch_pdl_cluster(score_select_kernel<2>, g2, b2, kSelCluster, smem, s, qr, mc, nb_max, sw, idx, cnt);
    case 3: return launch_pdl_cluster(score_select_kernel<3>, g2, b2, kSelCluster, smem, s, qr, mc, nb_max, sw, idx, cnt);
    case 4: return launch_pdl_cluster(score_select_kernel<4>, g2, b2, kSelCluster, smem, s, qr, mc, nb_max, sw, idx, cnt);
    case 5: return launch_pdl_cluster(score_select_kernel<5>, g2, b2, kSelCluster, smem, s, qr, mc, nb_max, sw, idx, cnt);
    case 6: return launch_pdl_cluster(score_select_kernel<6>, g2, b2, kSelCluster, smem, s, qr, mc, nb_max, sw, idx, cnt);
    case 7: return launch_pdl_cluster(score_select_kernel<7>, g2, b2, kSelCluster, smem, s, qr, mc, nb_max, sw, idx, cnt);
    default: return launch_pdl_cluster(score_select_kernel<8>, g2, b2, kSelCluster, smem, s, qr, mc, nb_max, sw, idx, cnt);
    }
}

}  // namespace iv2

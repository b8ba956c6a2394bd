// score_tc.cu -- block scoring and top-k for many query rows (prefill) on the 5th-generation tensor cores.
//
// Same definition as score.cu ("Tsinghua & ModelBest: MiniCPM4 technical details", "Model architecture:
// InfLLM v2", items 1-3): for query row (token t, head h) of KV group g the score of kernel j is
// z = scale * q . kern_j, LSE_h is the log-sum-exp of z over the kernels token t sees, a block's raw
// score is the max of z over its kernels, and the group score is S_b = sum_h exp(max_hb - LSE_h); the
// top-k of S plus the initial and local blocks is the token's block set.  Specialised for 16 query heads
// per KV group and head_dim 128.
//
// One CTA owns 16 consecutive tokens x the 16 heads of one KV group: two tiles of 128 query rows (A: the
// first 8 tokens, B: the next 8), each row one TMEM lane.  The kernel cache of the group streams twice
// through a 3-stage TMA ring, 128 kernels (32 blocks) per stage, and every stage feeds both tiles: two
// M = N = 128, K = 128 products S_A = Q_A . K^T and S_B = Q_B . K^T (Q in TMEM, kernels K-major in
// 128-byte-swizzled shared memory), so the kernel-cache bytes per token are half those of one tile:
//   pass 1: LSE of every row (online max / sum of 2^z, scores in log2 units);
//   pass 2: block maxima from the same scores, 2^(max - LSE), summed over the 16 heads of a token by
//           warp shuffles (a token's rows are 16 consecutive lanes) into S in shared memory.
// Then each reader warp selects the blocks of one token (warp_select_topk_hist).
// Warp roles: warp 0 issues the TMA loads, warp 1 (one thread) issues the MMAs, warps 2-17 read TMEM: one
// lane of each tile per thread, the four warps of a lane quarter each taking 32 of the 128 kernels.  The
// readers hand a stage's accumulators back right after loading them, so the next stage's MMAs overlap
// their arithmetic.  Every wait is bounded: after the limit the CTA records an error (g_score_tc_error)
// and skips its work.
#include "common.cuh"
#include "internal.h"
#include "select.cuh"
#include "tc.cuh"

namespace iv2 {

__device__ int g_score_tc_error = 0;

namespace {

constexpr int kSTile = 8;            // tokens per 128-row tile
constexpr int kSTok = 2 * kSTile;    // tokens per CTA
constexpr int kSG = 16;              // heads per KV group
constexpr int kSD = 128;             // head dim
constexpr int kSThreads = 576;       // 18 warps
constexpr int kSParts = 4;           // reader warps per TMEM lane quarter
constexpr int kSEpiThreads = 128 * kSParts;  // warps 2..17
constexpr int kSRing = 3;
constexpr int kSSlot = 32768;        // 128 kernel rows x 128 dims: two 64-dim atoms of 16 KB
constexpr int kSMaxNb = 1024;        // context blocks (64K keys)
constexpr uint32_t kSTmemCols = 512;  // S_A [0,128), S_B [128,256), Q_A [256,320), Q_B [320,384)
constexpr uint32_t kSColQ = 256;
constexpr int kSQOff = kSRing * kSSlot;  // Q tiles staged by TMA (2 x 32 KB), later the group scores S
constexpr int kSQBytes = 2 * 32768;

// the rest of the layout depends on nb_max (the pitch of S)
struct SLayout {
    int s_bytes, lse_off, ws_off, bytes;
    __host__ __device__ explicit SLayout(int nb_max)
    {
        s_bytes = kSTok * nb_max * 4;
        lse_off = kSQOff + (s_bytes > kSQBytes ? s_bytes : kSQBytes);  // [parts][256] max, [parts][256] sum
        ws_off = lse_off + 2 * kSParts * 256 * 4;                        // per reader warp: WarpSelectSmem
        bytes = ws_off + 4 * kSParts * (int)sizeof(WarpSelectSmem) + 1024;  // + alignment slack
    }
};

struct SBars {
    uint64_t q_full, q_tmem;
    uint64_t k_full[kSRing], k_empty[kSRing];
    uint64_t s_full[2], s_empty[2];  // per tile (A, B): accumulator ready / read back
    uint64_t drain;                  // the issuer's last MMAs
    uint64_t never;                  // nothing arrives on it: the wait a test drives to run out
    uint32_t tmem_base;
    int err;
};

__device__ __forceinline__ bool swait(uint64_t* bar, uint32_t parity, volatile int* err, uint32_t limit = 1u << 22)
{
    for (uint32_t i = 0; i < limit; ++i) {
        if (tc::mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u && *err) return false;
    }
    *err = 1;
    atomicOr(&g_score_tc_error, 1);
    return false;
}

// 32 scores of this thread's part of one row, scaled to log2 units; kernels at or past nkv are -inf
IV2_DEV void scaled_row(const uint32_t (&v)[32], int j0, int nkv, float sl2, float (&z)[32])
{
#pragma unroll
    for (int c = 0; c < 32; ++c) z[c] = j0 + c < nkv ? __uint_as_float(v[c]) * sl2 : neg_inf();
}

}  // namespace

template <int KW>
__global__ void __launch_bounds__(kSThreads, 1)
score_tc_kernel(QueryRows qr, const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kern,
                const __grid_constant__ CUtensorMap tm_kern_s, int nk_cap, MethodConsts mc, int nb_max,
                int32_t* __restrict__ idx, int32_t* __restrict__ cnt, unsigned test_wait_limit)
{
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = tc::align_smem_1024(smem_raw);
    __shared__ SBars bars;
    const SLayout lay(nb_max);
    float* Ssm = reinterpret_cast<float*>(smem + kSQOff);  // after Q has gone to TMEM
    float* hm_sm = reinterpret_cast<float*>(smem + lay.lse_off);  // [part][tile * 128 + row]
    float* hs_sm = hm_sm + kSParts * 256;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.y % qr.Hkv, b = blockIdx.y / qr.Hkv;
    // longest tiles first (later tokens see more kernels): the short ones fill the last wave
    const int t0 = (gridDim.x - 1 - blockIdx.x) * kSTok;
    const int T = q_len(qr, b);  // this sequence's queries (qr.T unless the batch is packed)
    if (t0 >= T) return;         // uniform over the CTA, before any barrier

    int n_max = 0;
    bool any_sparse = false;
#pragma unroll
    for (int tt = 0; tt < kSTok; ++tt)
        if (t0 + tt < T) {
            const int n = query_ctx(qr, b, t0 + tt);
            n_max = max(n_max, n);
            any_sparse |= n > mc.dense_len;
        }
    if (!any_sparse) {  // uniform over the CTA: dense rows only
        for (int tt = warp; tt < kSTok && t0 + tt < T; tt += kSThreads / 32) {
            const int n = query_ctx(qr, b, t0 + tt);
            const size_t row = (size_t)q_row(qr, b, t0 + tt) * qr.Hkv + g;
            warp_write_dense_row((n - 1) / kBlock, mc.kmax, idx + row * mc.kmax, cnt + row);
        }
        return;
    }
    const int nb = min((n_max - 1) / kBlock + 1, nb_max);
    const int ntiles = (nb + 31) / 32;  // 32 blocks (128 kernels) per stage
    // pass 1 reads every ls-th kernel (ls = 1: all of them) through tm_kern_s, 128 per stage
    const int ls = mc.lse_stride > 1 ? mc.lse_stride : 1;
    const int n1 = (nb + 32 * ls - 1) / (32 * ls);
    const int nq = n1 + ntiles;          // stages over both passes

    if (threadIdx.x == 0) {
        bars.err = 0;
        tc::mbar_init(&bars.q_full, 1);
        tc::mbar_init(&bars.q_tmem, 128);
        for (int i = 0; i < kSRing; ++i) {
            tc::mbar_init(&bars.k_full[i], 1);
            tc::mbar_init(&bars.k_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&bars.s_full[i], 1);
            tc::mbar_init(&bars.s_empty[i], kSEpiThreads);
        }
        tc::mbar_init(&bars.drain, 1);
        tc::mbar_init(&bars.never, 1);
        tc::fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(&bars.tmem_base, kSTmemCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = bars.tmem_base;
    volatile int* err = &bars.err;

    if (warp == 0) {
        // ---------------- TMA producer: both Q tiles once, then the kernel stages of both passes ----------------
        if (lane == 0) {
            tc::prefetch_tensormap(&tm_q);
            tc::prefetch_tensormap(&tm_kern);
            if (ls > 1) tc::prefetch_tensormap(&tm_kern_s);
            tc::mbar_arrive_expect_tx(&bars.q_full, kSQBytes);
#pragma unroll
            for (int tile = 0; tile < 2; ++tile) {
                const int zq = (int)q_row(qr, b, t0 + kSTile * tile);  // rows past the sequence are masked
                tc::tma_load_3d(smem + kSQOff + 32768 * tile, &tm_q, 0, g * kSG, zq, &bars.q_full);
                tc::tma_load_3d(smem + kSQOff + 32768 * tile + 16384, &tm_q, 64, g * kSG, zq, &bars.q_full);
            }
            const int zk = b * qr.Hkv + g;
            int issued = 0;  // stages whose copies are in flight or landed
            for (int q = 0; q < nq; ++q, ++issued) {
                const int s = q % kSRing, k = q / kSRing;
                if (k >= 1 && !swait(&bars.k_empty[s], (k - 1) & 1, err)) break;
                unsigned char* st = smem + s * kSSlot;
                // pass 1: rows 128 q .. of the strided view (kernels ls * row); pass 2: kernels 128 (q - n1) ..
                const CUtensorMap* map = q < n1 ? &tm_kern_s : &tm_kern;
                const int row0 = (q < n1 ? q : q - n1) * 128;
                tc::mbar_arrive_expect_tx(&bars.k_full[s], kSSlot);
                tc::tma_load_3d(st, map, 0, row0, zk, &bars.k_full[s]);
                tc::tma_load_3d(st + 16384, map, 64, row0, zk, &bars.k_full[s]);
            }
            // every copy this lane issued has landed before the CTA ends (on the normal path each one was
            // waited for already); after a wait ran out, the rest of the CTA no longer waits for them
            (void)tc::mbar_wait(&bars.q_full, 0, 1u << 22);
            for (int s = 0; s < kSRing && s < issued; ++s)
                (void)tc::mbar_wait(&bars.k_full[s], ((issued - 1 - s) / kSRing) & 1, 1u << 22);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer: S_A(q), S_B(q) = Q_A, Q_B . K(q)^T ----------------
        // (with a test limit, the first wait polls a barrier nothing arrives on instead)
        if (lane == 0 && (test_wait_limit ? swait(&bars.never, 0, err, test_wait_limit) : swait(&bars.q_tmem, 0, err))) {
            tc::tc_fence_after();
            constexpr uint32_t idesc = tc::idesc_bf16(128, 128, false);
            const uint32_t sbase = tc::smem_u32(smem);
            for (int q = 0; q < nq; ++q) {
                const int s = q % kSRing;
                if (!swait(&bars.k_full[s], (q / kSRing) & 1, err)) break;
                const uint32_t kb = sbase + s * kSSlot;
                bool fail = false;
#pragma unroll
                for (int tile = 0; tile < 2; ++tile) {
                    // tile's accumulator of stage q - 1 must have been read back
                    if (q >= 1 && !swait(&bars.s_empty[tile], (q - 1) & 1, err)) {
                        fail = true;
                        break;
                    }
                    tc::tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < kSD / 16; ++ks) {
                        const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
                        tc::mma_bf16_ts(tmem + 128 * tile, tmem + kSColQ + 64 * tile + 8 * ks,
                                        tc::desc_kmajor_sw128(kb + koff), idesc, ks > 0);
                    }
                    tc::mma_commit(&bars.s_full[tile]);
                }
                if (fail) break;
                tc::mma_commit(&bars.k_empty[s]);
            }
        }
        if (lane == 0) tc::mma_drain(&bars.drain);
    } else {
        // ---------------- TMEM readers: lane r of both tiles per thread, 32 columns per warp ----------------
        const int q4 = warp & 3, part = (warp - 2) >> 2;
        const int r = q4 * 32 + lane;  // row = token * 16 + head within a tile
        const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
        const float sl2 = mc.scale * kLog2e;
        int nkv[2], c_t[2], tt[2];
        bool valid[2];
#pragma unroll
        for (int tile = 0; tile < 2; ++tile) {
            tt[tile] = kSTile * tile + (r >> 4);
            const int t = t0 + tt[tile];
            valid[tile] = t < T;
            const int n = valid[tile] ? query_ctx(qr, b, t) : 0;
            nkv[tile] = min(num_kernels(n), nk_cap);
            c_t[tile] = n > 0 ? (n - 1) / kBlock : -1;
        }
        bool ok = swait(&bars.q_full, 0, err);
        if (part == 0) {
            // row r of both Q tiles (swizzled smem from TMA) -> TMEM columns [kSColQ + 64 tile, +64) as bf16 pairs
#pragma unroll
            for (int tile = 0; tile < 2; ++tile)
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    uint32_t w[32];
                    const unsigned char* qrow = smem + kSQOff + 32768 * tile + a * 16384 + r * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 v4 = *reinterpret_cast<const uint4*>(qrow + ((c ^ (r & 7)) << 4));
                        w[4 * c] = v4.x;
                        w[4 * c + 1] = v4.y;
                        w[4 * c + 2] = v4.z;
                        w[4 * c + 3] = v4.w;
                    }
                    tc::tmem_st32(lane_addr + kSColQ + 64 * tile + 32 * a, w);
                }
            tc::tmem_wait_st();
            tc::tc_fence_before();
            tc::mbar_arrive(&bars.q_tmem);
        }
        ok = __all_sync(0xffffffffu, ok);

        // ---- pass 1: LSE of both rows over their visible kernels (finite floor: no inf - inf) ----
        constexpr float kFloor = -1e30f;
        float m[2] = {kFloor, kFloor}, s[2] = {0.f, 0.f};
        for (int q = 0; q < n1 && ok; ++q) {
            const int i0 = 128 * q + 32 * part;  // strided rows: column c is kernel ls * (i0 + c)
#pragma unroll
            for (int tile = 0; tile < 2; ++tile) {
                ok = __all_sync(0xffffffffu, swait(&bars.s_full[tile], q & 1, err));
                if (!ok) break;
                tc::tc_fence_after();
                uint32_t v[32];
                tc::tmem_ld32(lane_addr + 128 * tile + 32 * part, v);
                tc::tmem_wait_ld();
                tc::tc_fence_before();
                tc::mbar_arrive(&bars.s_empty[tile]);
                float z[32], mx = kFloor;
                // visible: ls * (i0 + c) < nkv, i.e. i0 + c < ceil(nkv / ls)
                scaled_row(v, i0, (nkv[tile] + ls - 1) / ls, sl2, z);
#pragma unroll
                for (int c = 0; c < 32; ++c) mx = fmaxf(mx, z[c]);
                const float mn = fmaxf(m[tile], mx);
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < 32; ++c) acc[c & 3] += ex2_approx(z[c] - mn);  // one MUFU op, 2^-inf = 0
                s[tile] = s[tile] * ex2_approx(m[tile] - mn) + ((acc[0] + acc[1]) + (acc[2] + acc[3]));
                m[tile] = mn;
            }
        }
        // the four parts of each row -> LSE (every part forms the same value; named barrier over the readers)
#pragma unroll
        for (int tile = 0; tile < 2; ++tile) {
            hm_sm[part * 256 + 128 * tile + r] = m[tile];
            hs_sm[part * 256 + 128 * tile + r] = s[tile];
        }
        tc::named_bar_sync(1, kSEpiThreads);
        float lse_r[2];
#pragma unroll
        for (int tile = 0; tile < 2; ++tile) {
            float M = kFloor;
#pragma unroll
            for (int k2 = 0; k2 < kSParts; ++k2) M = fmaxf(M, hm_sm[k2 * 256 + 128 * tile + r]);
            float sum = 0.f;
#pragma unroll
            for (int k2 = 0; k2 < kSParts; ++k2)
                sum += hs_sm[k2 * 256 + 128 * tile + r] * exp2_fast(hm_sm[k2 * 256 + 128 * tile + r] - M);
            // the estimate scales the strided sum by ls (ls = 1: exact)
            lse_r[tile] = (M == kFloor) ? neg_inf() : M + __log2f(sum * (float)ls);
        }
        const bool overlap = mc.membership == 0;

        // ---- pass 2: block maxima -> 2^(max - LSE) -> summed over the token's 16 heads -> S ----
        float prev_last[2] = {neg_inf(), neg_inf()};  // part 0: the kernel before its first column
        for (int q = n1; q < nq && ok; ++q) {
            const int i = q - n1;
            const int j0 = 128 * i + 32 * part;
#pragma unroll
            for (int tile = 0; tile < 2; ++tile) {
                ok = __all_sync(0xffffffffu, swait(&bars.s_full[tile], q & 1, err));
                if (!ok) break;
                tc::tc_fence_after();
                uint32_t v[32];
                tc::tmem_ld32(lane_addr + 128 * tile + 32 * part, v);
                // parts 1-3: column 32 part - 1 precedes their first column; part 0: column 127 precedes the
                // next stage's first
                const uint32_t extra = tc::tmem_ld1(lane_addr + 128 * tile + (part ? 32 * part - 1 : 127));
                tc::tmem_wait_ld();
                tc::tc_fence_before();
                tc::mbar_arrive(&bars.s_empty[tile]);
                const float halo = part ? (j0 - 1 < nkv[tile] ? __uint_as_float(extra) * sl2 : neg_inf())
                                        : prev_last[tile];
                if (part == 0) prev_last[tile] = j0 + 127 < nkv[tile] ? __uint_as_float(extra) * sl2 : neg_inf();
                float z[32];
                scaled_row(v, j0, nkv[tile], sl2, z);
                // the 8 blocks of this part: 2^(max - LSE) of each, then the sums over the token's 16 heads
                // (8 independent shuffle chains, interleaved)
                float e[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    float bm = overlap ? fmaxf(fmaxf(z[4 * k], z[4 * k + 1]), fmaxf(z[4 * k + 2], z[4 * k + 3]))
                                       : fmaxf(fmaxf(z[4 * k], z[4 * k + 1]), z[4 * k + 2]);
                    if (overlap) bm = fmaxf(bm, k == 0 ? halo : z[4 * k - 1]);
                    e[k] = lse_r[tile] != neg_inf() ? ex2_approx(bm - lse_r[tile]) : 0.f;
                }
#pragma unroll
                for (int o = 1; o < 16; o <<= 1)
#pragma unroll
                    for (int k = 0; k < 8; ++k) e[k] += __shfl_xor_sync(0xffffffffu, e[k], o);
                if ((lane & 15) == 0 && valid[tile]) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int blk = 32 * i + 8 * part + k;
                        // a block scores only when one of its kernels is visible (same rule for every head)
                        int lo, hi;
                        block_kernel_range(blk, mc.membership, lo, hi);
                        if (blk <= c_t[tile] && blk < nb)
                            Ssm[tt[tile] * nb_max + blk] = max(lo, 0) < min(hi, nkv[tile]) ? e[k] : neg_inf();
                    }
                }
            }
        }
        // ---- selection: reader warp w takes token w - 2 ----
        tc::named_bar_sync(1, kSEpiThreads);
        ok = __all_sync(0xffffffffu, ok && !*err);
        const int ts = warp - 2;
        if (ok && t0 + ts < T) {
            const int tsel = t0 + ts;
            const int ns = query_ctx(qr, b, tsel);
            const int cs = (ns - 1) / kBlock;
            const size_t row = (size_t)q_row(qr, b, tsel) * qr.Hkv + g;
            if (ns <= mc.dense_len)
                warp_write_dense_row(cs, mc.kmax, idx + row * mc.kmax, cnt + row);
            else if (cs >= nb_max) {  // a context past the launch's max_ctx: no scores for it
                if (lane == 0) {
                    cnt[row] = 0;
                    atomicOr(&g_score_tc_error, 2);
                }
            } else
                warp_select_topk_hist<KW>(Ssm + ts * nb_max, cs, mc.init_blocks, mc.local_blocks, mc.topk, mc.kmax,
                                          idx + row * mc.kmax, cnt + row,
                                          reinterpret_cast<WarpSelectSmem*>(smem + lay.ws_off)[warp - 2]);
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kSTmemCols);
    }
}

// ---------------------------------------------------------------- host
bool score_tc_supported(const QueryRows& qr, int nb_max)
{
    return qr.D == kSD && qr.Hq / qr.Hkv == kSG && nb_max <= kSMaxNb;
}

template <int KW>
static cudaError_t score_tc_launch(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tks,
                                   const QueryRows& qr, int nk_cap, const MethodConsts& mc, int nb_max, int32_t* idx,
                                   int32_t* cnt, cudaStream_t s)
{
    const SLayout lay(nb_max);
    cudaError_t e = ensure_smem(score_tc_kernel<KW>, lay.bytes);
    if (e != cudaSuccess) return e;
    const dim3 grid((qr.T + kSTok - 1) / kSTok, qr.B * qr.Hkv);
    return launch_pdl(score_tc_kernel<KW>, grid, dim3(kSThreads), (size_t)lay.bytes, s, qr, tq, tk, tks, nk_cap, mc,
                      nb_max, idx, cnt, test_first_wait_limit());
}

cudaError_t launch_score_tc(const QueryRows& qr, const void* kern, int nk_cap, const MethodConsts& mc, int nb_max,
                            int32_t* idx, int32_t* cnt, cudaStream_t s)
{
    if (!score_tc_supported(qr, nb_max)) return cudaErrorNotSupported;
    CUtensorMap tq, tk, tks;
    const uint64_t row = (uint64_t)kSD * 2;
    if (!make_tma_map_bf16(&tq, qr.q, kSD, qr.Hq, (uint64_t)qr.q_rows, row, row * qr.Hq, kSG, kSTile) ||
        !make_tma_map_bf16(&tk, kern, kSD, (uint64_t)nk_cap, (uint64_t)qr.B * qr.Hkv, row, row * nk_cap, 128, 1))
        return cudaErrorNotSupported;
    // the LSE estimate's view: every ls-th kernel row (row stride ls rows; rows past nk_cap are outside the map)
    const int ls = mc.lse_stride > 1 ? mc.lse_stride : 1;
    if (ls == 1) tks = tk;
    else if (!make_tma_map_bf16(&tks, kern, kSD, (uint64_t)(nk_cap + ls - 1) / ls, (uint64_t)qr.B * qr.Hkv, row * ls,
                                row * nk_cap, 128, 1))
        return cudaErrorNotSupported;
    // keys per lane of the warp select: nb_max <= 32 KW
    if (nb_max <= 256) return score_tc_launch<8>(tq, tk, tks, qr, nk_cap, mc, nb_max, idx, cnt, s);
    if (nb_max <= 512) return score_tc_launch<16>(tq, tk, tks, qr, nk_cap, mc, nb_max, idx, cnt, s);
    return score_tc_launch<32>(tq, tk, tks, qr, nk_cap, mc, nb_max, idx, cnt, s);
}

int score_tc_error_flag_read_and_clear()
{
    int h = 0;
    if (cudaMemcpyFromSymbol(&h, g_score_tc_error, sizeof(int)) != cudaSuccess) return -1;
    if (h) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_score_tc_error, &zero, sizeof(int));
    }
    return h;
}

}  // namespace iv2

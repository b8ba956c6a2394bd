// attn_bwd_tc.cu -- dq of the block-sparse attention backward on the 5th-generation tensor cores.
//
// Same definition as attn_bwd.cu (the derivative of the forward's definition for a fixed selection; "Tsinghua
// & ModelBest: MiniCPM4 technical details", "Model architecture: InfLLM v2", item 3: the operators serve
// training as well as inference).  For a row (token t, head h) with key set K(t):
//   p_e = 2^(scale log2e q.k_e - lse log2e),  ds_e = p_e (dout . v_e - Dsum),  dq = scale sum_e ds_e k_e.
// Specialised for 16 query heads per KV group and head_dim 128.
//
// One CTA owns a 128-row tile (8 consecutive tokens x the 16 heads of one KV group) and walks the ascending
// union of its tokens' block sets, one 64-key block per step (a token reads a block only when it selected
// it; the other rows are masked for that block).  Per step:
//   S  [128 x 64]  = Q  . K^T      tcgen05.mma, A (Q) in TMEM, B (K) K-major in 128B-swizzled smem
//   dP [128 x 64]  = dO . V^T      the same with dO and V
//   dS             = P (dP - Dsum) eight warps, one TMEM lane (row) per thread, 32 keys each; dS goes back
//                                  to TMEM as bf16 pairs over its own S buffer
//   dQ [128 x 128] += dS . K       A (dS) in TMEM, B (K) MN-major in smem, dQ in TMEM
// S and dP are double-buffered, so the products of step p + 1 run while the warps form dS of step p.  No
// online softmax is needed: the forward's lse normalises every step directly.
// Warp roles: warp 0 loads Q and dO once and K per step, warp 10 loads V per step (TMA, one lane each, 3-deep
// rings), warps 1, 11 and 12 (one thread each) issue the S, dP and dQ MMAs (one thread issues a tcgen05.mma
// every ~107 cycles; three keep the tensor pipe fed), warps 2-9 form dS and write dq.  Every wait is bounded: after
// the limit the CTA records an error (g_bwd_tc_error), skips the rest of its work, frees its TMEM and exits.
#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace iv2 {

__device__ int g_bwd_tc_error = 0;

namespace {

constexpr int kTok = 8;         // tokens per tile
constexpr int kG = 16;          // heads per KV group
constexpr int kD = 128;         // head dim
constexpr int kThreads = 416;   // 13 warps
constexpr int kMaxBlk = 4096;   // context blocks (256K keys)
constexpr int kWords = kMaxBlk / 32;
constexpr int kRing = 3;
constexpr int kSlot = 16384;    // one 64-key block of K or V: two d-halves x 64 rows x 128 B
constexpr int kKOff = 0;
constexpr int kVOff = kKOff + kRing * kSlot;
constexpr int kQOff = kVOff + kRing * kSlot;   // Q tile: two d-halves x 128 rows x 128 B
constexpr int kDoOff = kQOff + 32768;          // dO tile, same layout
constexpr int kBitsOff = kDoOff + 32768;       // [kTok][kWords] uint32
constexpr int kListOff = kBitsOff + kTok * kWords * 4;  // uint16 block ids
constexpr int kSmemBytes = kListOff + kMaxBlk * 2 + 1024;  // + alignment slack
// TMEM: dQ [0,128), S [128,256) (two 64-column buffers), dP [256,384) (two), Q [384,448), dO [448,512)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 128, kColDP = 256, kColQ = 384, kColDO = 448;

struct Bars {
    uint64_t qd_full, qd_tmem;
    uint64_t k_full[kRing], k_empty[kRing], v_full[kRing], v_empty[kRing];
    uint64_t s_full[2], ds_full[2], dq_done[2];
    uint64_t drain[3];  // the S, dP and dQ issuers' last MMAs
    uint32_t tmem_base;
    int n_union;
    int err;
};

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* err)
{
    for (uint32_t i = 0; i < (1u << 22); ++i) {
        if (tc::mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u && *err) return false;
    }
    *err = 1;
    atomicOr(&g_bwd_tc_error, 1);
    return false;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
bwd_dq_tc_kernel(QueryRows qr, const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                 const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, int Lcap,
                 const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt, MethodConsts mc, int dense_all,
                 const float* __restrict__ lse, const float* __restrict__ dsum, float* __restrict__ dq)
{
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = tc::align_smem_1024(smem_raw);
    __shared__ Bars bars;
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + kBitsOff);
    uint16_t* list = reinterpret_cast<uint16_t*>(smem + kListOff);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = qr.T;
    const int g = blockIdx.y % qr.Hkv, b = blockIdx.y / qr.Hkv;
    const int t0 = (gridDim.x - 1 - blockIdx.x) * kTok;  // longest tiles first

    // ---- union of the tile's block sets, as one bitmap per token and an ascending list ----
    int cmax = 0;
#pragma unroll
    for (int tt = 0; tt < kTok; ++tt)
        if (t0 + tt < T) cmax = max(cmax, (query_ctx(qr, b, t0 + tt) - 1) / kBlock);
    const int nwords = min(cmax / 32 + 1, kWords);
    for (int i = threadIdx.x; i < kTok * kWords; i += kThreads) bits[i] = 0u;
    if (threadIdx.x == 0) {
        bars.err = 0;
        bars.n_union = 0;
    }
    __syncthreads();
    for (int item = threadIdx.x; item < kTok * max(mc.kmax, nwords); item += kThreads) {
        const int tt = item % kTok, e = item / kTok;
        const int t = t0 + tt;
        if (t >= T) continue;
        const int n = query_ctx(qr, b, t);
        const int c = (n - 1) / kBlock;
        if (dense_all || n <= mc.dense_len) {
            if (e < nwords) {  // every block 0..c
                const int lo = e * 32, hi = min(c + 1, lo + 32);
                if (hi > lo) bits[tt * kWords + e] = (hi - lo == 32) ? 0xffffffffu : ((1u << (hi - lo)) - 1u);
            }
        } else if (e < mc.kmax) {
            const size_t row = ((size_t)b * T + t) * qr.Hkv + g;
            if (e < min(cnt[row], mc.kmax)) {
                const int blk = idx[row * mc.kmax + e];
                if (blk >= 0 && blk * kBlock < n) atomicOr(&bits[tt * kWords + (blk >> 5)], 1u << (blk & 31));
            }
        }
    }
    __syncthreads();
    if (warp == 0) {
        int base = 0;
        for (int w0 = 0; w0 < nwords; w0 += 32) {
            const int w = w0 + lane;
            uint32_t u = 0u;
            if (w < nwords)
#pragma unroll
                for (int tt = 0; tt < kTok; ++tt) u |= bits[tt * kWords + w];
            const int cntw = __popc(u);
            int incl = cntw;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            int pos = base + incl - cntw;
            while (u) {
                const int bit = __ffs(u) - 1;
                list[pos++] = (uint16_t)(w * 32 + bit);
                u &= u - 1u;
            }
            base += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) bars.n_union = base;
    }
    if (threadIdx.x == 0) {
        tc::mbar_init(&bars.qd_full, 1);
        tc::mbar_init(&bars.qd_tmem, 128);
        for (int i = 0; i < kRing; ++i) {
            tc::mbar_init(&bars.k_full[i], 1);
            tc::mbar_init(&bars.k_empty[i], 2);  // K(p) is read by S(p) and dQ(p): one commit from each issuer
            tc::mbar_init(&bars.v_full[i], 1);
            tc::mbar_init(&bars.v_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&bars.s_full[i], 2);  // S(p) and dP(p) both landed: one commit from each issuer
            tc::mbar_init(&bars.ds_full[i], 256);
            tc::mbar_init(&bars.dq_done[i], 1);
        }
        for (int i = 0; i < 3; ++i) tc::mbar_init(&bars.drain[i], 1);
        tc::fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(&bars.tmem_base, kTmemCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const int U = bars.n_union;
    const uint32_t tmem = bars.tmem_base;
    volatile int* err = &bars.err;
    const uint32_t sK = tc::smem_u32(smem + kKOff);
    const uint32_t sV = tc::smem_u32(smem + kVOff);

    if (warp == 0 || warp == 10) {
        // ---------------- TMA producers: warp 0 Q, dO once and K per step; warp 10 V per step ----------------
        if (warp == 0 && lane == 0) {
            tc::prefetch_tensormap(&tm_q);
            tc::prefetch_tensormap(&tm_do);
            tc::prefetch_tensormap(&tm_k);
            tc::mbar_arrive_expect_tx(&bars.qd_full, 4 * 16384);
            const int zq = b * T + t0;
#pragma unroll
            for (int a = 0; a < 2; ++a) {
                tc::tma_load_3d(smem + kQOff + a * 16384, &tm_q, 64 * a, g * kG, zq, &bars.qd_full);
                tc::tma_load_3d(smem + kDoOff + a * 16384, &tm_do, 64 * a, g * kG, zq, &bars.qd_full);
            }
            for (int p = 0; p < U; ++p) {
                const int s = p % kRing, k = p / kRing;
                if (k >= 1 && !wait_bar(&bars.k_empty[s], (k - 1) & 1, err)) break;
                unsigned char* st = smem + kKOff + s * kSlot;
                const int z = b * Lcap + (int)list[p] * kBlock;
                tc::mbar_arrive_expect_tx(&bars.k_full[s], kSlot);
                tc::tma_load_3d(st, &tm_k, 0, g, z, &bars.k_full[s]);
                tc::tma_load_3d(st + 8192, &tm_k, 64, g, z, &bars.k_full[s]);
            }
        } else if (warp == 10 && lane == 0) {
            tc::prefetch_tensormap(&tm_v);
            for (int p = 0; p < U; ++p) {
                const int s = p % kRing, k = p / kRing;
                if (k >= 1 && !wait_bar(&bars.v_empty[s], (k - 1) & 1, err)) break;
                unsigned char* st = smem + kVOff + s * kSlot;
                const int z = b * Lcap + (int)list[p] * kBlock;
                tc::mbar_arrive_expect_tx(&bars.v_full[s], kSlot);
                tc::tma_load_3d(st, &tm_v, 0, g, z, &bars.v_full[s]);
                tc::tma_load_3d(st + 8192, &tm_v, 64, g, z, &bars.v_full[s]);
            }
        }
    } else if (warp == 1 || warp == 11) {
        // ---------------- S issuer (warp 1) and dP issuer (warp 11) ----------------
        // S(p) and dP(p) go to buffers p & 1.  S(p) overwrites dS(p - 2), so it waits until dQ(p - 2) has
        // completed; dP(p) overwrites dP(p - 2), which the dS warps loaded before they signalled dS(p - 2)
        const bool is_s = warp == 1;
        if (lane == 0 && wait_bar(&bars.qd_tmem, 0, err)) {
            tc::tc_fence_after();
            constexpr uint32_t idesc_s = tc::idesc_bf16(128, kBlock, false);
            for (int p = 0; p < U; ++p) {
                const int s = p % kRing, sb = p & 1;
                if (p >= 2 && !wait_bar(is_s ? &bars.dq_done[sb] : &bars.ds_full[sb], ((p - 2) >> 1) & 1, err))
                    break;
                if (!wait_bar(is_s ? &bars.k_full[s] : &bars.v_full[s], (p / kRing) & 1, err)) break;
                tc::tc_fence_after();
                const uint32_t ob = (is_s ? sK : sV) + s * kSlot;
                const uint32_t d_t = tmem + (is_s ? kColS : kColDP) + kBlock * sb;
                const uint32_t a_t = tmem + (is_s ? kColQ : kColDO);
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * 8192 + (ks & 3) * 32;
                    tc::mma_bf16_ts(d_t, a_t + 8 * ks, tc::desc_kmajor_sw128(ob + off), idesc_s, ks > 0);
                }
                tc::mma_commit(&bars.s_full[sb]);
                tc::mma_commit(is_s ? &bars.k_empty[s] : &bars.v_empty[s]);
            }
        }
        if (lane == 0) tc::mma_drain(&bars.drain[is_s ? 0 : 1]);
    } else if (warp == 12) {
        // ---------------- dQ issuer: dQ += dS(v) . K(v), dS(v) in the first 32 columns of S buffer v & 1 ----------
        if (lane == 0) {
            constexpr uint32_t idesc_q = tc::idesc_bf16(128, kD, true);
            for (int v = 0; v < U; ++v) {
                const int db = v & 1, s = v % kRing;
                if (!wait_bar(&bars.ds_full[db], (v >> 1) & 1, err)) break;
                if (!wait_bar(&bars.k_full[s], (v / kRing) & 1, err)) break;  // landed before S(v): no wait
                tc::tc_fence_after();
                const uint32_t kb = sK + s * kSlot;
#pragma unroll
                for (int ks = 0; ks < kBlock / 16; ++ks)
                    tc::mma_bf16_ts(tmem, tmem + kColS + kBlock * db + 8 * ks,
                                    tc::desc_mnmajor_sw128(kb + ks * 2048, 8192), idesc_q, (v > 0 || ks > 0));
                tc::mma_commit(&bars.dq_done[db]);
                tc::mma_commit(&bars.k_empty[s]);
            }
            tc::mma_drain(&bars.drain[2]);
        }
    } else if (warp >= 2 && warp <= 9) {
        // ---------------- dS and dq: one TMEM lane (query row) per thread, 32 keys of each step ----------------
        // warps w and w + 4 (2 <= w <= 5) share the lane quarter w & 3: half 0 takes keys 0..31 of the block,
        // half 1 keys 32..63; they meet at a named barrier of their own on every step before dS overwrites S
        const int q4 = warp & 3, half = (warp - 2) >> 2;
        const int r = q4 * 32 + lane;  // row = token * 16 + head
        const int tt = r >> 4, hh = r & 15;
        const int t = t0 + tt;
        const bool valid = t < T;
        const int n = valid ? query_ctx(qr, b, t) : 0;
        const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
        const uint32_t pair_bar = 1 + q4;
        const float sl2 = mc.scale * kLog2e;
        const size_t head = ((size_t)b * T + (valid ? t : 0)) * qr.Hq + g * kG + hh;
        float lse2 = __int_as_float(0x7f800000), dd = 0.f;  // +inf: this row's p is 0
        if (valid) {
            const float lv = lse[head];
            if (lv > neg_inf() && lv < __int_as_float(0x7f800000)) lse2 = lv * kLog2e;
            dd = dsum[head];
        }
        bool ok = wait_bar(&bars.qd_full, 0, err);
        if (half == 0) {
            // this row of Q and of dO (swizzled smem from TMA) -> TMEM as bf16 pairs
#pragma unroll
            for (int m2 = 0; m2 < 2; ++m2)
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    uint32_t w[32];
                    const unsigned char* src = smem + (m2 ? kDoOff : kQOff) + a * 16384 + r * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 v4 = *reinterpret_cast<const uint4*>(src + ((c ^ (r & 7)) << 4));
                        w[4 * c] = v4.x;
                        w[4 * c + 1] = v4.y;
                        w[4 * c + 2] = v4.z;
                        w[4 * c + 3] = v4.w;
                    }
                    tc::tmem_st32(lane_addr + (m2 ? kColDO : kColQ) + 32 * a, w);
                }
            tc::tmem_wait_st();
            tc::tc_fence_before();
            tc::mbar_arrive(&bars.qd_tmem);
        }
        ok = __all_sync(0xffffffffu, ok);
        for (int p = 0; p < U; ++p) {
            const int sb = p & 1;
            if (ok) ok = wait_bar(&bars.s_full[sb], (p >> 1) & 1, err);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) tc::tc_fence_after();
            const int blk = list[p];
            const bool sel = valid && ((bits[tt * kWords + (blk >> 5)] >> (blk & 31)) & 1u);
            const int nv = sel ? min(32, n - blk * kBlock - 32 * half) : 0;  // may be <= 0
            const bool any_sel = __any_sync(0xffffffffu, sel);
            uint32_t sv[32], pv[32];
            if (ok && any_sel) {
                tc::tmem_ld32(lane_addr + kColS + kBlock * sb + 32 * half, sv);
                tc::tmem_ld32(lane_addr + kColDP + kBlock * sb + 32 * half, pv);
                tc::tmem_wait_ld();
            }
            // both halves' S loads are complete past this barrier, so dS may overwrite S columns 0..31
            tc::named_bar_sync(pair_bar, 64);
            if (ok) {
                uint32_t w[16];
                if (any_sel) {
#pragma unroll
                    for (int j2 = 0; j2 < 16; ++j2) {
                        const int j = 2 * j2;
                        const float p0 = j < nv ? ex2_approx(__uint_as_float(sv[j]) * sl2 - lse2) : 0.f;
                        const float p1 = j + 1 < nv ? ex2_approx(__uint_as_float(sv[j + 1]) * sl2 - lse2) : 0.f;
                        w[j2] = pack_bf16(p0 * (__uint_as_float(pv[j]) - dd), p1 * (__uint_as_float(pv[j + 1]) - dd));
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) w[j] = 0u;
                }
                tc::tmem_st16(lane_addr + kColS + kBlock * sb + 16 * half, w);
                tc::tmem_wait_st();
                tc::tc_fence_before();
                tc::mbar_arrive(&bars.ds_full[sb]);
            }
        }
        ok = __all_sync(0xffffffffu, ok);
        if (ok && U > 0) ok = wait_bar(&bars.dq_done[(U - 1) & 1], ((U - 1) >> 1) & 1, err);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc::tc_fence_after();
            float* drow = dq + head * kD + 64 * half;
#pragma unroll 1
            for (int c4 = 0; c4 < 2; ++c4) {
                uint32_t o[32];
                tc::tmem_ld32(lane_addr + 64 * half + 32 * c4, o);
                tc::tmem_wait_ld();
                if (U == 0) {  // no token of the tile selected a block: dQ was never written, dq is 0
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = 0u;
                }
                if (valid) {
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<float4*>(drow + 32 * c4 + 4 * c) =
                            make_float4(__uint_as_float(o[4 * c]) * mc.scale, __uint_as_float(o[4 * c + 1]) * mc.scale,
                                        __uint_as_float(o[4 * c + 2]) * mc.scale,
                                        __uint_as_float(o[4 * c + 3]) * mc.scale);
                }
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------- host
bool bwd_dq_tc_supported(const QueryRows& qr)
{
    return qr.D == kD && qr.Hq / qr.Hkv == kG && (qr.max_ctx - 1) / kBlock + 1 <= kMaxBlk;
}

cudaError_t launch_bwd_dq_tc(const QueryRows& qr, const void* k, const void* v, int Lcap, const int32_t* idx,
                             const int32_t* cnt, const MethodConsts& mc, bool dense_all, const float* lse,
                             const float* dsum, const void* dout, float* dq, cudaStream_t s)
{
    if (!bwd_dq_tc_supported(qr)) return cudaErrorNotSupported;
    CUtensorMap tq, tdo, tk, tv;
    const uint64_t row = (uint64_t)kD * 2;
    if (!make_tma_map_bf16(&tq, qr.q, kD, qr.Hq, (uint64_t)qr.B * qr.T, row, row * qr.Hq, kG, kTok) ||
        !make_tma_map_bf16(&tdo, dout, kD, qr.Hq, (uint64_t)qr.B * qr.T, row, row * qr.Hq, kG, kTok) ||
        !make_tma_map_bf16(&tk, k, kD, qr.Hkv, (uint64_t)qr.B * Lcap, row, row * qr.Hkv, 1, kBlock) ||
        !make_tma_map_bf16(&tv, v, kD, qr.Hkv, (uint64_t)qr.B * Lcap, row, row * qr.Hkv, 1, kBlock))
        return cudaErrorNotSupported;
    cudaError_t e = ensure_smem(bwd_dq_tc_kernel, kSmemBytes);
    if (e != cudaSuccess) return e;
    const dim3 grid((qr.T + kTok - 1) / kTok, qr.B * qr.Hkv);
    return launch_pdl(bwd_dq_tc_kernel, grid, dim3(kThreads), (size_t)kSmemBytes, s, qr, tq, tdo, tk, tv, Lcap, idx,
                      cnt, mc, dense_all ? 1 : 0, lse, dsum, dq);
}

// =====================================================================================================
// dk, dv: one 64-key block against 8-token tiles of its token list
// =====================================================================================================
//   S   [128 rows x 64 keys]   = Q . K^T            A (Q) and B (K) K-major in smem
//   dP  [128 x 64]             = dO . V^T
//   P, dS                      rows in TMEM -> bf16 tiles in smem (four warps, one row per thread)
//   dV^T [128 dims x 64 keys] += dO^T . P           A (dO) MN-major, B (P) MN-major, in TMEM
//   dK^T [128 dims x 64 keys] += Q^T . dS           the same with Q and dS
// S and dP are double-buffered, so tile i + 1's products run while the warps form tile i's P and dS.  Warp 1
// issues S and dP, warp 6 the dV / dK sums (one thread issues a tcgen05.mma every ~107 cycles; two keep the
// tensor pipe busier).  A work item's sums go to dk / dv by fp32 atomics (one TMEM lane = one head dimension
// per thread).
namespace {

constexpr int kKvThreads = 224;   // warp 0 TMA, warps 1 and 6 MMA, warps 2-5 P / dS and the flush
constexpr int kKvItemTokens = 256;  // tokens per work item (the list builder's chunk)
constexpr int kKvTile = 16384;    // one 64-key block of K or V
constexpr int kKvQd = 32768;      // one 8-token tile of Q or dO: two d-halves x 128 rows x 128 B
constexpr int kKvKOff = 0;
constexpr int kKvVOff = kKvKOff + kKvTile;
constexpr int kKvQOff = kKvVOff + kKvTile;       // [2] x (Q | dO)
constexpr int kKvPOff = kKvQOff + 4 * kKvQd;     // P tile: 128 rows x 64 keys bf16 (128 B rows, swizzled)
constexpr int kKvSOff = kKvPOff + 16384;         // dS tile
constexpr int kKvTokOff = kKvSOff + 16384;       // [2][8] token ids of the Q / dO buffers
constexpr int kKvSmemBytes = kKvTokOff + 64 + 1024;
// TMEM: S [0,128) (two 64-column buffers), dP [128,256) (two), dV^T [256,320), dK^T [320,384)
constexpr uint32_t kKvCols = 512, kKvColS = 0, kKvColDP = 128, kKvColDV = 256, kKvColDK = 320;

struct KvBars {
    uint64_t kv_full, kv_free, qd_full[2], qd_free[2], s_full[2], pd_full, pd_free, acc_done, acc_free;
    uint64_t drain[2];  // the S / dP and dV / dK issuers' last MMAs
    uint32_t tmem_base;
    int err;
};

}  // namespace

__global__ void __launch_bounds__(kKvThreads, 1)
bwd_dkdv_tc_kernel(QueryRows qr, const __grid_constant__ CUtensorMap tm_q1, const __grid_constant__ CUtensorMap tm_do1,
                   const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, int Lcap,
                   MethodConsts mc, int nb, const float* __restrict__ lse, const float* __restrict__ dsum,
                   const int* __restrict__ counts, const int* __restrict__ offsets, const int* __restrict__ tokens,
                   const int* __restrict__ nitems, const int* __restrict__ item_list,
                   const int* __restrict__ item_start, int cap, float* __restrict__ dk, float* __restrict__ dv)
{
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = tc::align_smem_1024(smem_raw);
    __shared__ KvBars bars;
    int* tok_sm = reinterpret_cast<int*>(smem + kKvTokOff);  // [2][8]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = qr.T;
    const int n_items = *nitems;

    if (threadIdx.x == 0) {
        bars.err = 0;
        tc::mbar_init(&bars.kv_full, 1);
        tc::mbar_init(&bars.kv_free, 1);
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&bars.qd_full[i], 1);
            tc::mbar_init(&bars.qd_free[i], 2);  // Q / dO are read by both issuers' products
            tc::mbar_init(&bars.s_full[i], 1);
        }
        tc::mbar_init(&bars.pd_full, 128);
        tc::mbar_init(&bars.pd_free, 1);
        tc::mbar_init(&bars.acc_done, 1);
        tc::mbar_init(&bars.acc_free, 128);
        tc::mbar_init(&bars.drain[0], 1);
        tc::mbar_init(&bars.drain[1], 1);
        tc::fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(&bars.tmem_base, kKvCols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = bars.tmem_base;
    volatile int* err = &bars.err;
    const uint32_t sbase = tc::smem_u32(smem);

    // every role walks the same items and tiles; the counters give each barrier's phase
    if (warp == 0) {
        // ---------------- TMA: the block's K and V per item, Q and dO rows of 8 tokens per tile ----------------
        if (lane == 0) {
            tc::prefetch_tensormap(&tm_q1);
            tc::prefetch_tensormap(&tm_do1);
            tc::prefetch_tensormap(&tm_k);
            tc::prefetch_tensormap(&tm_v);
            int n_item = 0, n_tile = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++n_item) {
                const int l = item_list[item], start = item_start[item];
                const int b = l / (qr.Hkv * nb), g = (l / nb) % qr.Hkv, kb = l % nb;
                const int ntok = min(min(kKvItemTokens, counts[l] - start), cap - offsets[l] - start);
                const int* toks = tokens + offsets[l] + start;
                if (n_item >= 1 && !(ok = wait_bar(&bars.kv_free, (n_item - 1) & 1, err))) break;
                tc::mbar_arrive_expect_tx(&bars.kv_full, 2 * kKvTile);
                const int z = b * Lcap + kb * kBlock;
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    tc::tma_load_3d(smem + kKvKOff + a * 8192, &tm_k, 64 * a, g, z, &bars.kv_full);
                    tc::tma_load_3d(smem + kKvVOff + a * 8192, &tm_v, 64 * a, g, z, &bars.kv_full);
                }
                const int ntiles = ntok > 0 ? (ntok + kTok - 1) / kTok : 0;
                for (int i = 0; i < ntiles; ++i, ++n_tile) {
                    const int qb = n_tile & 1, use = n_tile >> 1;
                    if (use >= 1 && !(ok = wait_bar(&bars.qd_free[qb], (use - 1) & 1, err))) break;
                    // token slots past the list repeat its first token (finite rows; their p is masked to 0); the
                    // ids are stored before the arrive, whose release orders them for the readers
                    unsigned char* qt = smem + kKvQOff + qb * 2 * kKvQd;
                    int tsl[kTok];
#pragma unroll
                    for (int s = 0; s < kTok; ++s) {
                        const int j = i * kTok + s;
                        tsl[s] = toks[j < ntok ? j : i * kTok];
                        tok_sm[qb * kTok + s] = j < ntok ? tsl[s] : -1;
                    }
                    tc::mbar_arrive_expect_tx(&bars.qd_full[qb], 2 * kKvQd);
#pragma unroll
                    for (int s = 0; s < kTok; ++s) {
                        const int t = tsl[s];
#pragma unroll
                        for (int a = 0; a < 2; ++a) {
                            tc::tma_load_3d(qt + a * 16384 + s * 2048, &tm_q1, 64 * a, g * kG, b * T + t, &bars.qd_full[qb]);
                            tc::tma_load_3d(qt + kKvQd + a * 16384 + s * 2048, &tm_do1, 64 * a, g * kG, b * T + t,
                                            &bars.qd_full[qb]);
                        }
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- S / dP issuer ----------------
        // S, dP of tile ctr into buffers ctr & 1.  That buffer held tile ctr - 2, whose reads are ordered before
        // this product: Q / dO of tile ctr land only after both issuers freed the buffer for tile ctr - 2, and
        // warp 6 freed it after dV / dK of P(ctr - 2), which the warps wrote after reading S(ctr - 2)
        if (lane == 0) {
            constexpr uint32_t idesc_s = tc::idesc_bf16_ab(128, kBlock, false, false);
            int n_item = 0, n_tile = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++n_item) {
                const int l = item_list[item], start = item_start[item];
                const int ntok = min(min(kKvItemTokens, counts[l] - start), cap - offsets[l] - start);
                const int ntiles = ntok > 0 ? (ntok + kTok - 1) / kTok : 0;
                if (!(ok = wait_bar(&bars.kv_full, n_item & 1, err))) break;
                for (int i = 0; i < ntiles; ++i) {
                    const int ctr = n_tile + i, sb = ctr & 1;
                    if (!(ok = wait_bar(&bars.qd_full[sb], (ctr >> 1) & 1, err))) break;
                    tc::tc_fence_after();
                    const uint32_t qa = sbase + kKvQOff + sb * 2 * kKvQd, da = qa + kKvQd;
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks) {
                        const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                        const uint32_t boff = (ks >> 2) * 8192 + (ks & 3) * 32;
                        tc::mma_bf16_ss(tmem + kKvColS + kBlock * sb, tc::desc_kmajor_sw128(qa + off),
                                        tc::desc_kmajor_sw128(sbase + kKvKOff + boff), idesc_s, ks > 0);
                        tc::mma_bf16_ss(tmem + kKvColDP + kBlock * sb, tc::desc_kmajor_sw128(da + off),
                                        tc::desc_kmajor_sw128(sbase + kKvVOff + boff), idesc_s, ks > 0);
                    }
                    tc::mma_commit(&bars.s_full[sb]);
                    tc::mma_commit(&bars.qd_free[sb]);
                }
                if (!ok) break;
                n_tile += ntiles;
                tc::mma_commit(&bars.kv_free);  // only S and dP read the item's K and V
            }
            tc::mma_drain(&bars.drain[0]);
        }
    } else if (warp == 6) {
        // ---------------- dV / dK issuer: dV^T += dO^T P, dK^T += Q^T dS per tile ----------------
        if (lane == 0) {
            constexpr uint32_t idesc_t = tc::idesc_bf16_ab(128, kBlock, true, true);
            int n_item = 0, n_tile = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++n_item) {
                const int l = item_list[item], start = item_start[item];
                const int ntok = min(min(kKvItemTokens, counts[l] - start), cap - offsets[l] - start);
                const int ntiles = ntok > 0 ? (ntok + kTok - 1) / kTok : 0;
                // the flush of the previous item's sums must be done before this item's first accumulation
                if (n_item >= 1 && !(ok = wait_bar(&bars.acc_free, (n_item - 1) & 1, err))) break;
                for (int i = 0; i < ntiles; ++i) {
                    const int ctr = n_tile + i;
                    if (!(ok = wait_bar(&bars.qd_full[ctr & 1], (ctr >> 1) & 1, err))) break;
                    if (!(ok = wait_bar(&bars.pd_full, ctr & 1, err))) break;
                    tc::tc_fence_after();
                    const uint32_t qa = sbase + kKvQOff + (ctr & 1) * 2 * kKvQd, da = qa + kKvQd;
#pragma unroll
                    for (int ks = 0; ks < 128 / 16; ++ks) {  // over the tile's 128 rows
                        tc::mma_bf16_ss(tmem + kKvColDV, tc::desc_mnmajor_sw128(da + ks * 2048, 16384),
                                        tc::desc_mnmajor_sw128(sbase + kKvPOff + ks * 2048, 16384), idesc_t,
                                        (i > 0 || ks > 0));
                        tc::mma_bf16_ss(tmem + kKvColDK, tc::desc_mnmajor_sw128(qa + ks * 2048, 16384),
                                        tc::desc_mnmajor_sw128(sbase + kKvSOff + ks * 2048, 16384), idesc_t,
                                        (i > 0 || ks > 0));
                    }
                    tc::mma_commit(&bars.pd_free);
                    tc::mma_commit(&bars.qd_free[ctr & 1]);
                }
                if (!ok) break;
                n_tile += ntiles;
                tc::mma_commit(&bars.acc_done);
            }
            tc::mma_drain(&bars.drain[1]);
        }
    } else if (warp >= 2 && warp <= 5) {
        // ---------------- P, dS (one query row per thread) and the flush (one head dimension per thread) ----------
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;  // tile row = token slot * 16 + head; in the flush: head dimension
        const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
        const float sl2 = mc.scale * kLog2e;
        int n_item = 0, n_tile = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++n_item) {
            const int l = item_list[item], start = item_start[item];
            const int b = l / (qr.Hkv * nb), g = (l / nb) % qr.Hkv, kb = l % nb;
            const int ntok = min(min(kKvItemTokens, counts[l] - start), cap - offsets[l] - start);
            const int ntiles = ntok > 0 ? (ntok + kTok - 1) / kTok : 0;
            for (int i = 0; i < ntiles; ++i, ++n_tile) {
                const int sb = n_tile & 1;
                // the token ids of this tile's Q / dO buffer (n_tile & 1, as S) were stored before the TMA warp's
                // arrive on qd_full: waiting on it orders those stores before the reads below.  It completed
                // before s_full and cannot run ahead (its next phase needs this tile's products done).
                if (ok) ok = wait_bar(&bars.qd_full[sb], (n_tile >> 1) & 1, err);
                if (ok) ok = wait_bar(&bars.s_full[sb], (n_tile >> 1) & 1, err);
                ok = __all_sync(0xffffffffu, ok);
                if (ok) tc::tc_fence_after();
                const int t = ok ? tok_sm[sb * kTok + (r >> 4)] : -1;
                const bool valid = t >= 0;
                const size_t head = ((size_t)b * T + (valid ? t : 0)) * qr.Hq + g * kG + (r & 15);
                const int n = valid ? query_ctx(qr, b, t) : 0;
                float lse2 = __int_as_float(0x7f800000), dd = 0.f;
                if (valid) {
                    const float lv = lse[head];
                    if (lv > neg_inf() && lv < __int_as_float(0x7f800000)) lse2 = lv * kLog2e;
                    dd = dsum[head];
                }
                const int nv = valid ? min(kBlock, n - kb * kBlock) : 0;  // keys of the block this row sees
                uint32_t sv[64], pv[64];
                if (ok) {
                    tc::tmem_ld32(lane_addr + kKvColS + kBlock * sb, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                    tc::tmem_ld32(lane_addr + kKvColS + kBlock * sb + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
                    tc::tmem_ld32(lane_addr + kKvColDP + kBlock * sb, *reinterpret_cast<uint32_t(*)[32]>(&pv[0]));
                    tc::tmem_ld32(lane_addr + kKvColDP + kBlock * sb + 32, *reinterpret_cast<uint32_t(*)[32]>(&pv[32]));
                    tc::tmem_wait_ld();
                }
                // the P / dS tiles of the previous tile must have been read by its products
                if (ok && n_tile >= 1) ok = wait_bar(&bars.pd_free, (n_tile - 1) & 1, err);
                ok = __all_sync(0xffffffffu, ok);
                if (ok) {
                    unsigned char* prow = smem + kKvPOff + r * 128;
                    unsigned char* drow = smem + kKvSOff + r * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        uint32_t pw[4], dw[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int j = 8 * c + 2 * e;
                            const float p0 = j < nv ? ex2_approx(__uint_as_float(sv[j]) * sl2 - lse2) : 0.f;
                            const float p1 = j + 1 < nv ? ex2_approx(__uint_as_float(sv[j + 1]) * sl2 - lse2) : 0.f;
                            pw[e] = pack_bf16(p0, p1);
                            dw[e] = pack_bf16(p0 * (__uint_as_float(pv[j]) - dd), p1 * (__uint_as_float(pv[j + 1]) - dd));
                        }
                        const int sw = (c ^ (r & 7)) << 4;
                        *reinterpret_cast<uint4*>(prow + sw) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
                        *reinterpret_cast<uint4*>(drow + sw) = make_uint4(dw[0], dw[1], dw[2], dw[3]);
                    }
                    tc::fence_proxy_async_smem();  // generic-proxy tile writes -> visible to the tensor core
                    tc::tc_fence_before();
                    tc::mbar_arrive(&bars.pd_full);
                }
            }
            // this item's dV^T, dK^T: lane r is head dimension r; 64 columns are the block's keys
            if (ok) ok = wait_bar(&bars.acc_done, n_item & 1, err);
            ok = __all_sync(0xffffffffu, ok);
            if (ok && ntiles > 0) {
                tc::tc_fence_after();
#pragma unroll 1
                for (int m2 = 0; m2 < 2; ++m2) {
                    float* dst = m2 ? dk : dv;
                    const float mul = m2 ? mc.scale : 1.f;
#pragma unroll 1
                    for (int h2 = 0; h2 < 2; ++h2) {
                        uint32_t a[32];
                        tc::tmem_ld32(lane_addr + (m2 ? kKvColDK : kKvColDV) + 32 * h2, a);
                        tc::tmem_wait_ld();
#pragma unroll 4
                        for (int j = 0; j < 32; ++j) {
                            const int key = kb * kBlock + 32 * h2 + j;
                            if (key < Lcap)
                                atomicAdd(dst + (((size_t)b * Lcap + key) * qr.Hkv + g) * kD + r,
                                          __uint_as_float(a[j]) * mul);
                        }
                    }
                }
            }
            if (ok) {
                tc::tc_fence_before();
                tc::mbar_arrive(&bars.acc_free);
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kKvCols);
    }
}

bool bwd_dkdv_tc_supported(const QueryRows& qr)
{
    return qr.D == kD && qr.Hq / qr.Hkv == kG;
}

cudaError_t launch_bwd_dkdv_tc(const QueryRows& qr, const void* k, const void* v, int Lcap, const MethodConsts& mc,
                               int nb, const float* lse, const float* dsum, const void* dout, const int* counts,
                               const int* offsets, const int* tokens, const int* nitems, const int* item_list,
                               const int* item_start, int cap, int max_items, float* dk, float* dv, cudaStream_t s)
{
    if (!bwd_dkdv_tc_supported(qr)) return cudaErrorNotSupported;
    CUtensorMap tq, tdo, tk, tv;
    const uint64_t row = (uint64_t)kD * 2;
    if (!make_tma_map_bf16(&tq, qr.q, kD, qr.Hq, (uint64_t)qr.B * qr.T, row, row * qr.Hq, kG, 1) ||
        !make_tma_map_bf16(&tdo, dout, kD, qr.Hq, (uint64_t)qr.B * qr.T, row, row * qr.Hq, kG, 1) ||
        !make_tma_map_bf16(&tk, k, kD, qr.Hkv, (uint64_t)qr.B * Lcap, row, row * qr.Hkv, 1, kBlock) ||
        !make_tma_map_bf16(&tv, v, kD, qr.Hkv, (uint64_t)qr.B * Lcap, row, row * qr.Hkv, 1, kBlock))
        return cudaErrorNotSupported;
    cudaError_t e = ensure_smem(bwd_dkdv_tc_kernel, kKvSmemBytes);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const int grid = max(1, min(nsm, max_items));
    return launch_pdl(bwd_dkdv_tc_kernel, dim3(grid), dim3(kKvThreads), (size_t)kKvSmemBytes, s, qr, tq, tdo, tk, tv,
                      Lcap, mc, nb, lse, dsum, counts, offsets, tokens, nitems, item_list, item_start, cap, dk, dv);
}

int bwd_tc_error_flag_read_and_clear()
{
    int h = 0;
    if (cudaMemcpyFromSymbol(&h, g_bwd_tc_error, sizeof(int)) != cudaSuccess) return -1;
    if (h) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_bwd_tc_error, &zero, sizeof(int));
    }
    return h;
}

}  // namespace iv2

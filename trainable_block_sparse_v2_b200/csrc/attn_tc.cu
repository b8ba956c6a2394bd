// attn_tc.cu -- block-sparse prefill attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Same definition as attn.cu (MiniCPM4 technical details, InfLLM v2 overview: only the selected context
// blocks take part in attention; "Model architecture: InfLLM v2" item 2: the query heads of one GQA group
// share the block set).  Instantiated for G = 2, 4, 8 or 16 query heads per KV group and head_dim d = 64 or
// 128 (not G = 2 with d = 128, whose token bitmaps and rings exceed shared memory).
//
// One CTA owns a 128-row tile = 128 / G consecutive query tokens x the G heads of one KV group, and walks the
// ascending union of those tokens' selected blocks two blocks (128 keys) at a time (a token attends to a
// block only when it selected it; other rows of the tile are masked for that block).  Per step:
//   S[128 x 128] = Q[128 x d] . K^T         tcgen05.mma kind::f16, A (Q) and B (K) K-major in 128B-swizzled
//                                            smem, fp32 accumulator in TMEM (three S buffers)
//   P            = online softmax of S       four warps, one TMEM lane (= one query row) per thread; P goes
//                                            back to TMEM as bf16 pairs over its own S buffer; the output
//                                            is rescaled only when a row's max grows by more than 2^8 (exact:
//                                            O and the row sum share the reference max)
//   O[128 x d] += P[128 x 128] . V           A (P) in TMEM, B (V) MN-major in smem, O in TMEM
// The step chain P(p) -> PV(p) -> S(p + 3) -> P(p + 3) spans three steps: with three S buffers the softmax
// of step p overlaps the MMAs of steps p + 1 and p + 2, and 128-key steps halve the number of MMA
// instructions and pipeline hand-offs per key.
// Warp roles: warps 0 and 10 issue TMA loads (Q once and K per step; V per step) into rings, one lane each,
// warp 1 (one thread) issues the S MMAs and warp 11 (one thread) the PV MMAs, so that a late P does not hold
// back the next scores; warps 2-9 run the softmax and the epilogue, two warps per TMEM lane quarter, each on
// one of the step's two blocks.
// Producer/consumer hand-offs use mbarriers; MMA completion is signalled with tcgen05.commit.  Every wait
// is bounded: after the limit the CTA records an error (g_tc_error) and skips the rest of its work; each
// producer then waits (bounded) for the copies it issued and each MMA issuer for its MMAs, and the CTA frees
// its TMEM and exits with nothing in flight.
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace iv2 {

__device__ int g_tc_error = 0;

namespace {

constexpr int kThreads = 384;     // 12 warps
constexpr int kMaxBlk = 4096;     // context blocks (256K keys)
constexpr int kWords = kMaxBlk / 32;
constexpr int kStepKeys = 128;       // two 64-key blocks per pipeline step
constexpr uint32_t kTmemCols = 512;  // O [0,d), S buffers [128,256), [256,384), [384,512); P(step) overwrites
                                     // the first 64 columns of its own S buffer
constexpr uint32_t kColS = 128;
constexpr int kNS = 3;               // S buffers: the scores of step p + 2 are computed while P(p) is formed
constexpr int kRing = 3;             // K ring depth, in steps of 128 keys

// dynamic shared memory layout (base aligned to 1024 B).  K and V stream through separate rings so each
// can be refilled as soon as its own MMA has consumed it; Q stays in shared memory as the A operand of every
// S MMA.  A 128-B swizzle atom holds 64 dims of 128 rows.  V is needed only once P of its step is formed, two
// steps after its slot was freed, so at d 128 a 2-deep V ring leaves room for Q.
template <int G, int D>
struct TcShape {
    static constexpr int kTok = 128 / G;                     // tokens per tile
    static constexpr int kAtoms = D / 64;                    // 64-dim atoms of a row
    static constexpr int kSlot = kAtoms * 16384;             // one step of K or V: atoms x 128 key rows x 128 B
    static constexpr int kVRing = D == 128 ? 2 : 3;          // V ring depth
    static constexpr int kKOff = 0;
    static constexpr int kVOff = kKOff + kRing * kSlot;
    static constexpr int kQOff = kVOff + kVRing * kSlot;       // Q: atoms x 128 rows x 128 B
    static constexpr int kBitsOff = kQOff + kSlot;             // [kTok][kWords] uint32
    static constexpr int kListOff = kBitsOff + kTok * kWords * 4;  // uint16 block ids
    // + alignment slack; at least 116 KB, so that two CTAs never share an SM: each allocates all 512 TMEM columns
    static constexpr int kNeed = kListOff + kMaxBlk * 2 + 1024;
    static constexpr int kSmemBytes = kNeed > 116 * 1024 ? kNeed : 116 * 1024;
    static_assert(G * kTok == 128 && (D == 64 || D == 128), "128-row tiles of whole tokens, d 64 or 128");
    static_assert(kSmemBytes <= 227 * 1024 - 4096, "dynamic + static shared memory of one CTA");
};

struct Bars {
    uint64_t q_full;
    uint64_t k_full[kRing], k_empty[kRing], v_full[kRing], v_empty[kRing];
    uint64_t s_full[kNS], p_full[kNS], o_done[kNS];
    uint64_t drain[2];  // the S and PV issuers' last MMAs
    uint64_t never;     // nothing arrives on it: the wait a test drives to run out
    uint32_t tmem_base;
    int n_union;
    int err;
    float xm[2][2][128];  // [step parity][half][row]: the two softmax halves' partial maxima, then sums
};

// sm_100 paired fp32 arithmetic (two lanes of a 64-bit register pair per instruction, each rounded as the
// scalar op) and the three-input maximum
__device__ __forceinline__ unsigned long long f2(float lo, float hi)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_split(unsigned long long v, float& lo, float& hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b, unsigned long long c)
{
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ unsigned long long add2(unsigned long long a, unsigned long long b)
{
    unsigned long long d;
    asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float max3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* err,
                                         uint32_t limit = 1u << 22)
{
    for (uint32_t i = 0; i < limit; ++i) {
        if (tc::mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u && *err) return false;
    }
    *err = 1;
    atomicOr(&g_tc_error, 1);
    return false;
}

}  // namespace

template <int G, int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(QueryRows qr, const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, KvRows kr, const int32_t* __restrict__ idx,
               const int32_t* __restrict__ cnt, MethodConsts mc, int dense_all, __nv_bfloat16* __restrict__ out,
               float* __restrict__ lse, unsigned test_wait_limit)
{
    using Sh = TcShape<G, D>;
    constexpr int kTok = Sh::kTok, kSlot = Sh::kSlot, kKOff = Sh::kKOff, kVOff = Sh::kVOff, kQOff = Sh::kQOff;
    constexpr int kVRing = Sh::kVRing;
    constexpr int kBitsOff = Sh::kBitsOff, kListOff = Sh::kListOff;
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = tc::align_smem_1024(smem_raw);
    __shared__ Bars bars;
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + kBitsOff);
    uint16_t* list = reinterpret_cast<uint16_t*>(smem + kListOff);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.y % qr.Hkv, b = blockIdx.y / qr.Hkv;
    // longest tiles first (later tokens attend to more blocks): the short ones fill the last wave
    const int t0 = (gridDim.x - 1 - blockIdx.x) * kTok;
    const int Tb = q_len(qr, b);  // this sequence's queries (T unless the batch is packed)
    if (t0 >= Tb) return;         // uniform over the CTA, before any barrier

    // ---- union of the tile's block sets, as one bitmap per token and an ascending list ----
    int cmax = 0;
#pragma unroll
    for (int tt = 0; tt < kTok; ++tt)
        if (t0 + tt < Tb) cmax = max(cmax, (query_ctx(qr, b, t0 + tt) - 1) / kBlock);
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
        if (t >= Tb) continue;
        const int n = query_ctx(qr, b, t);
        const int c = (n - 1) / kBlock;
        if (dense_all || n <= mc.dense_len) {
            if (e < nwords) {  // every block 0..c
                const int lo = e * 32, hi = min(c + 1, lo + 32);
                if (hi > lo) bits[tt * kWords + e] = (hi - lo == 32) ? 0xffffffffu : ((1u << (hi - lo)) - 1u);
            }
        } else if (e < mc.kmax) {
            const size_t row = (size_t)q_row(qr, b, t) * qr.Hkv + g;
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
        tc::mbar_init(&bars.q_full, 1);
        for (int i = 0; i < kRing; ++i) {
            tc::mbar_init(&bars.k_full[i], 1);
            tc::mbar_init(&bars.k_empty[i], 1);
            tc::mbar_init(&bars.v_full[i], 1);
            tc::mbar_init(&bars.v_empty[i], 1);
        }
        for (int i = 0; i < kNS; ++i) {
            tc::mbar_init(&bars.s_full[i], 1);
            tc::mbar_init(&bars.p_full[i], 256);
            tc::mbar_init(&bars.o_done[i], 1);
        }
        tc::mbar_init(&bars.drain[0], 1);
        tc::mbar_init(&bars.drain[1], 1);
        tc::mbar_init(&bars.never, 1);
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

    const int NP = (U + 1) / 2;  // pipeline steps; an odd last block is paired with a masked copy of itself
    if (warp == 0 || warp == 10) {
        // ---------------- TMA producers: warp 0 streams K (and Q first), warp 10 streams V ----------------
        // (one lane each, in separate warps: two spinning lanes of one warp would take turns)
        if (warp == 0 && lane == 0) {
            tc::prefetch_tensormap(&tm_q);
            tc::prefetch_tensormap(&tm_k);
            tc::mbar_arrive_expect_tx(&bars.q_full, kSlot);
            const int zq = (int)q_row(qr, b, t0);  // rows past this sequence are masked (or zero-filled)
#pragma unroll
            for (int a = 0; a < Sh::kAtoms; ++a)
                tc::tma_load_3d(smem + kQOff + a * 16384, &tm_q, 64 * a, g * G, zq, &bars.q_full);
            int issued = 0;  // steps whose K copies are in flight or landed
            for (int p = 0; p < NP; ++p, ++issued) {
                const int s = p % kRing, k = p / kRing;
                if (k >= 1 && !wait_bar(&bars.k_empty[s], (k - 1) & 1, err)) break;
                unsigned char* st = smem + kKOff + s * kSlot;
                tc::mbar_arrive_expect_tx(&bars.k_full[s], kSlot);
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    // key rows [64 i, 64 i + 64) of the step, each 64-dim atom of 128 rows apart; an unmapped
                    // page starts a block before row 0, which the tensor map fills with zeros
                    const long zr = kv_block_row(kr, b, (int)list[min(2 * p + i, U - 1)]);
                    const int z = zr >= 0 ? (int)zr : -kBlock;
#pragma unroll
                    for (int a = 0; a < Sh::kAtoms; ++a)
                        tc::tma_load_3d(st + a * 16384 + i * 8192, &tm_k, 64 * a, g, z, &bars.k_full[s]);
                }
            }
            // every copy this lane issued has landed before the CTA ends (on the normal path each one was
            // waited for already); after a wait ran out, the rest of the CTA no longer waits for them
            (void)tc::mbar_wait(&bars.q_full, 0, 1u << 22);
            for (int s = 0; s < kRing && s < issued; ++s)  // stage s last took step s + kRing ((issued-1-s)/kRing)
                (void)tc::mbar_wait(&bars.k_full[s], ((issued - 1 - s) / kRing) & 1, 1u << 22);
        } else if (warp == 10 && lane == 0) {
            tc::prefetch_tensormap(&tm_v);
            int issued = 0;
            for (int p = 0; p < NP; ++p, ++issued) {
                const int s = p % kVRing, k = p / kVRing;
                if (k >= 1 && !wait_bar(&bars.v_empty[s], (k - 1) & 1, err)) break;
                unsigned char* st = smem + kVOff + s * kSlot;
                tc::mbar_arrive_expect_tx(&bars.v_full[s], kSlot);
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const long zr = kv_block_row(kr, b, (int)list[min(2 * p + i, U - 1)]);
                    const int z = zr >= 0 ? (int)zr : -kBlock;
#pragma unroll
                    for (int a = 0; a < Sh::kAtoms; ++a)
                        tc::tma_load_3d(st + a * 16384 + i * 8192, &tm_v, 64 * a, g, z, &bars.v_full[s]);
                }
            }
            for (int s = 0; s < kVRing && s < issued; ++s)
                (void)tc::mbar_wait(&bars.v_full[s], ((issued - 1 - s) / kVRing) & 1, 1u << 22);
        }
    } else if (warp == 1) {
        // ---------------- S issuer ----------------
        // S(p) overwrites the buffer of P(p - 3): it waits until PV(p - 3), issued by warp 11, has completed.
        // With a test limit, the first wait polls a barrier nothing arrives on instead of Q's
        if (lane == 0 && (test_wait_limit ? wait_bar(&bars.never, 0, err, test_wait_limit)
                                          : wait_bar(&bars.q_full, 0, err))) {
            tc::tc_fence_after();
            constexpr uint32_t idesc_s = tc::idesc_bf16(128, kStepKeys, false);
            const uint32_t sQ = tc::smem_u32(smem + kQOff);
            for (int p = 0; p < NP; ++p) {
                // S(p) = Q . [K_a ; K_b]^T into S buffer p % kNS, both operands K-major in shared memory
                const int s = p % kRing, sb = p % kNS;
                if (p >= kNS && !wait_bar(&bars.o_done[sb], ((p - kNS) / kNS) & 1, err)) break;
                if (!wait_bar(&bars.k_full[s], (p / kRing) & 1, err)) break;
                tc::tc_fence_after();
                const uint32_t d_s = tmem + kColS + kStepKeys * sb;
                const uint32_t kbase = sK + s * kSlot;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
                    tc::mma_bf16_ss(d_s, tc::desc_kmajor_sw128(sQ + koff), tc::desc_kmajor_sw128(kbase + koff),
                                    idesc_s, ks > 0);
                }
                tc::mma_commit(&bars.s_full[sb]);
                tc::mma_commit(&bars.k_empty[s]);
            }
        }
        if (lane == 0) tc::mma_drain(&bars.drain[0]);
    } else if (warp == 11) {
        // ---------------- PV issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idesc_o = tc::idesc_bf16(128, D, true);
            for (int v = 0; v < NP; ++v) {
                // O += P(v) . [V_a ; V_b], P(v) in the first 64 columns of S buffer v % kNS
                const int pv = v % kNS, sv = v % kVRing;
                if (!wait_bar(&bars.p_full[pv], (v / kNS) & 1, err)) break;
                if (!wait_bar(&bars.v_full[sv], (v / kVRing) & 1, err)) break;
                tc::tc_fence_after();
                const uint32_t vbase = sV + sv * kSlot;
#pragma unroll
                for (int ks = 0; ks < kStepKeys / 16; ++ks)
                    tc::mma_bf16_ts(tmem, tmem + kColS + kStepKeys * pv + 8 * ks,
                                    tc::desc_mnmajor_sw128(vbase + ks * 2048, 16384), idesc_o, (v > 0 || ks > 0));
                tc::mma_commit(&bars.o_done[pv]);
                tc::mma_commit(&bars.v_empty[sv]);
            }
            tc::mma_drain(&bars.drain[1]);
        }
    } else if (warp >= 2 && warp <= 9) {
        // ---------------- softmax + epilogue: one TMEM lane (query row) per thread, one block of each step ----
        // warps w and w + 4 (2 <= w <= 5) share the lane quarter w & 3: half 0 takes the step's first block
        // (keys 0..63), half 1 its second (keys 64..127); they exchange row maxima and sums in shared memory
        // under a named barrier of their own, and every barrier is reached by both on every step
        const int q4 = warp & 3, half = (warp - 2) >> 2;
        const int r = q4 * 32 + lane;  // row = token * G + head
        const int tt = r / G, hh = r % G;
        const int t = t0 + tt;
        const bool valid = t < Tb;
        const int n = valid ? query_ctx(qr, b, t) : 0;
        const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
        const uint32_t pair_bar = 1 + q4;
        const float sl2 = mc.scale * kLog2e;
        float m_ref = neg_inf(), l = 0.f;
        bool ok = true;
        for (int p = 0; p < NP; ++p) {
            const int sb = p % kNS;
            if (ok) ok = wait_bar(&bars.s_full[sb], (p / kNS) & 1, err);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) tc::tc_fence_after();
            // this half's block of the step, whether this row's token selected it, and its keys in it
            const int blk_a = list[2 * p];
            const bool has_b = 2 * p + 1 < U;
            const int blk = (half && has_b) ? list[2 * p + 1] : blk_a;
            const bool sel = valid && (half == 0 || has_b) && ((bits[tt * kWords + (blk >> 5)] >> (blk & 31)) & 1u);
            const int nv = sel ? min(kBlock, n - blk * kBlock) : 0;
            const uint32_t srow = lane_addr + kColS + kStepKeys * sb;
            const bool any_sel = __any_sync(0xffffffffu, sel);
            // raw scores of this half's 64 keys (both TMEM loads in flight together); keys this row does not
            // attend to are -inf.  The scale is applied later, inside the exponent's FFMA: with sl2 > 0 the
            // maximum of the scaled scores is sl2 times the maximum of the raw ones
            float x[64];
            float mx = neg_inf();
            if (ok && any_sel) {
                uint32_t sv[64];
                tc::tmem_ld32(srow + 64 * half, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                tc::tmem_ld32(srow + 64 * half + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
                tc::tmem_wait_ld();
                if (__all_sync(0xffffffffu, nv == kBlock)) {  // every row of the warp sees the whole block
#pragma unroll
                    for (int j = 0; j < 64; ++j) x[j] = __uint_as_float(sv[j]);
                } else {
#pragma unroll
                    for (int j = 0; j < 64; ++j) x[j] = j < nv ? __uint_as_float(sv[j]) : neg_inf();
                }
                // the maximum of 64 in 32 three-input steps: 64 -> 22 -> 8 -> 3 -> 1
                float m22[22];
#pragma unroll
                for (int i = 0; i < 21; ++i) m22[i] = max3(x[i], x[i + 21], x[i + 42]);
                m22[21] = x[63];
                float m8[8];
#pragma unroll
                for (int i = 0; i < 7; ++i) m8[i] = max3(m22[i], m22[i + 7], m22[i + 14]);
                m8[7] = m22[21];
                mx = max3(max3(m8[0], m8[1], m8[2]), max3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
                mx *= sl2;  // log2 units (-inf stays -inf)
            }
            // double-buffered by step parity: a half can be at most one step ahead of its partner here
            bars.xm[p & 1][half][r] = mx;
            // both halves' S loads are complete past this barrier, so P may overwrite S columns 0..63
            tc::named_bar_sync(pair_bar, 64);
            mx = fmaxf(mx, bars.xm[p & 1][half ^ 1][r]);
            const bool rescale = mx > m_ref + 8.f;  // mx is -inf for a row that selected neither block
            const float new_ref = rescale ? mx : m_ref;
            // identical in both halves: O is zero until the row has a finite reference
            const float alpha = (rescale && m_ref != neg_inf()) ? exp2_fast(m_ref - new_ref) : 1.f;
            if (ok && __any_sync(0xffffffffu, alpha != 1.f)) {
                // every PV so far must have landed before this half of O is rewritten
                if (p >= 1) ok = wait_bar(&bars.o_done[(p - 1) % kNS], ((p - 1) / kNS) & 1, err) && ok;
                ok = __all_sync(0xffffffffu, ok);
                if (ok) {
#pragma unroll 1
                    for (int c4 = 0; c4 < D / 64; ++c4) {  // this half's d / 2 columns of O
                        uint32_t o[32];
                        tc::tmem_ld32(lane_addr + (D / 2) * half + 32 * c4, o);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                        tc::tmem_st32(lane_addr + (D / 2) * half + 32 * c4, o);
                    }
                    tc::tmem_wait_st();
                }
            }
            l *= alpha;
            m_ref = new_ref;
            if (ok) {
                // P = 2^(x - m_ref) for this half's 64 keys, bf16 pairs into S columns [32 half, 32 half + 32)
                uint32_t w[32];
                if (any_sel) {
                    // 2^(sl2 s - m_ref) in one FFMA per key; a row that did not select the block (or has no
                    // finite reference yet) gets 2^-inf = 0
                    const float mneg = (sel && m_ref != neg_inf()) ? -m_ref : neg_inf();
                    // the exponents of a key pair in one paired FMA, the row sums in four paired accumulators
                    const unsigned long long sl2x2 = f2(sl2, sl2), mnegx2 = f2(mneg, mneg);
                    unsigned long long ps2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                    for (int j2 = 0; j2 < 32; ++j2) {
                        float e0, e1;
                        f2_split(fma2(f2(x[2 * j2], x[2 * j2 + 1]), sl2x2, mnegx2), e0, e1);
                        const float p0 = ex2_approx(e0), p1 = ex2_approx(e1);
                        ps2[j2 & 3] = add2(ps2[j2 & 3], f2(p0, p1));
                        w[j2] = pack_bf16(p0, p1);
                    }
                    float s0, s1, s2, s3;
                    f2_split(add2(ps2[0], ps2[1]), s0, s1);
                    f2_split(add2(ps2[2], ps2[3]), s2, s3);
                    l += (s0 + s1) + (s2 + s3);
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) w[j] = 0u;
                }
                tc::tmem_st32(srow + 32 * half, w);
                tc::tmem_wait_st();
                tc::tc_fence_before();
                tc::mbar_arrive(&bars.p_full[sb]);
            }
        }
        // the row sum over both halves
        tc::named_bar_sync(pair_bar, 64);  // every read of xm for the maxima is done
        bars.xm[0][half][r] = l;
        tc::named_bar_sync(pair_bar, 64);
        const float lt = l + bars.xm[0][half ^ 1][r];
        ok = __all_sync(0xffffffffu, ok);
        if (ok && NP > 0) ok = wait_bar(&bars.o_done[(NP - 1) % kNS], ((NP - 1) / kNS) & 1, err);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc::tc_fence_after();
            const float inv = lt > 0.f ? 1.f / lt : 0.f;
            __nv_bfloat16* orow = out + ((size_t)q_row(qr, b, valid ? t : 0) * qr.Hq + g * G + hh) * D + (D / 2) * half;
#pragma unroll 1
            for (int c4 = 0; c4 < D / 64; ++c4) {
                uint32_t o[32];
                tc::tmem_ld32(lane_addr + (D / 2) * half + 32 * c4, o);
                tc::tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            w[e] = pack_bf16(__uint_as_float(o[c * 8 + 2 * e]) * inv,
                                             __uint_as_float(o[c * 8 + 2 * e + 1]) * inv);
                        *reinterpret_cast<uint4*>(orow + c4 * 32 + c * 8) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
            if (valid && lse && half == 0)
                lse[(size_t)q_row(qr, b, t) * qr.Hq + g * G + hh] = lt > 0.f ? (m_ref + __log2f(lt)) * kLn2 : neg_inf();
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
namespace {

template <int G, int D>
cudaError_t attn_tc_launch(const QueryRows& qr, const void* k, const void* v, const KvRows& kr, const int32_t* idx,
                           const int32_t* cnt, const MethodConsts& mc, bool dense_all, void* out, float* lse,
                           cudaStream_t s)
{
    using Sh = TcShape<G, D>;
    CUtensorMap tq, tk, tv;
    const uint64_t row = (uint64_t)D * 2;
    if (!make_tma_map_bf16(&tq, qr.q, D, qr.Hq, (uint64_t)qr.q_rows, row, row * qr.Hq, G, Sh::kTok) ||
        !make_tma_map_bf16(&tk, k, D, qr.Hkv, (uint64_t)kr.rows, row, row * qr.Hkv, 1, kBlock) ||
        !make_tma_map_bf16(&tv, v, D, qr.Hkv, (uint64_t)kr.rows, row, row * qr.Hkv, 1, kBlock))
        return cudaErrorNotSupported;
    auto kfn = attn_tc_kernel<G, D>;
    cudaError_t e = ensure_smem(kfn, Sh::kSmemBytes);
    if (e != cudaSuccess) return e;
    const dim3 grid((qr.T + Sh::kTok - 1) / Sh::kTok, qr.B * qr.Hkv);
    return launch_pdl(kfn, grid, dim3(kThreads), (size_t)Sh::kSmemBytes, s, qr, tq, tk, tv, kr, idx, cnt, mc,
                      dense_all ? 1 : 0, static_cast<__nv_bfloat16*>(out), lse, test_first_wait_limit());
}

}  // namespace

bool attn_tc_supported(const QueryRows& qr)
{
    if (qr.Hkv <= 0 || qr.Hq % qr.Hkv != 0 || (qr.max_ctx - 1) / kBlock + 1 > kMaxBlk) return false;
    const int G = qr.Hq / qr.Hkv;
    if (qr.D == 64) return G == 2 || G == 4 || G == 8 || G == 16;
    return qr.D == 128 && (G == 4 || G == 8 || G == 16);
}

cudaError_t launch_attn_rows_tc(const QueryRows& qr, const void* k, const void* v, const KvRows& kr,
                                const int32_t* idx, const int32_t* cnt, const MethodConsts& mc, bool dense_all,
                                void* out, float* lse, cudaStream_t s)
{
    if (!attn_tc_supported(qr)) return cudaErrorNotSupported;
#define IV2_TC(GG, DD)                                                                                           \
    if (qr.Hq / qr.Hkv == GG && qr.D == DD) return attn_tc_launch<GG, DD>(qr, k, v, kr, idx, cnt, mc, dense_all, out, lse, s)
    IV2_TC(16, 128);
    IV2_TC(8, 128);
    IV2_TC(4, 128);
    IV2_TC(16, 64);
    IV2_TC(8, 64);
    IV2_TC(4, 64);
    IV2_TC(2, 64);
#undef IV2_TC
    return cudaErrorNotSupported;
}

int tc_error_flag_read_and_clear()
{
    int h = 0;
    if (cudaMemcpyFromSymbol(&h, g_tc_error, sizeof(int)) != cudaSuccess) return -1;
    if (h) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(int));
    }
    return h;
}

}  // namespace iv2

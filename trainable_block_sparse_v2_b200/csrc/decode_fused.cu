// decode_fused.cu -- one decode step of InfLLM v2 (block scoring, top-k, sparse attention) in one kernel.
//
// Same definitions as score.cu and attn.cu ("Tsinghua & ModelBest: MiniCPM4 technical details", "Model
// architecture: InfLLM v2", items 1-3; efficiency evaluation: a decode step reads a constant number of
// blocks plus the slowly growing kernel representations).  A thread-block cluster of CL CTAs owns one
// (sequence, query, KV group) row; CTA `rank` owns the context blocks [rank * bpc, (rank + 1) * bpc).
//
//   1. scan: the CTA streams the kernel rows of its blocks (4 per block) through a 3-stage ring of bulk
//      copies, 32 blocks per stage, and scores them on mma.sync with the G <= 16 heads as MMA rows; each
//      warp takes two 8-kernel tiles of a stage at once.  Per lane it keeps an online (max, sum 2^z) of
//      each head; block maxima go to shared memory by atomicMax on order-preserving keys.  Under the
//      overlapping-window rule a block also takes the last kernel of the block before it; for the CTA's
//      first block that kernel belongs to the CTA before, which adds it by a remote atomicMax.  Scores
//      are in log2 units (scale * log2 e folded in).
//   2. every CTA pushes its (max, sum) partials to all CTAs; after a cluster barrier each forms LSE_h
//      and the group score S = sum_h 2^(max_h - LSE_h) of its blocks, and pushes S to all CTAs.
//   3. selection: after a second barrier every CTA runs the same bucket select (select.cuh) on the whole
//      row, so the block list needs no broadcast; the leader (rank 0) writes idx / cnt.
//   4. attention: the CTA streams the K and V tiles of entries rank, rank + CL, ... through a 3-stage TMA
//      ring (128-byte swizzle, one producer thread); warp w takes keys [8w, 8w + 8) of every block (QK^T
//      on m16n8k16, PV on m16n8k8) with an online softmax; the eight warp states are merged in shared
//      memory.
//   5. combine: each CTA pushes its (O, m, l) of head h to CTA h % CL; after a third barrier that CTA
//      merges the CL partials and writes the output row.
// The footprint (about 112 KB of shared memory) lets two CTAs share an SM, so eight 16-CTA clusters are
// resident at once.  Every 2^x here has x <= 0 (a difference from a running or final maximum) or -inf,
// so the hardware ex2.approx (one MUFU op, tiny results flushed to zero) serves throughout.
#include <atomic>

#include <cooperative_groups.h>

#include "attn_warp.cuh"
#include "common.cuh"
#include "internal.h"
#include "select.cuh"
#include "tc.cuh"

namespace cg = cooperative_groups;

namespace iv2 {

namespace {

constexpr int kFThreads = 256;                          // 8 warps
constexpr int kFWarps = kFThreads / 32;
constexpr int kFChunkBlocks = 32;                       // blocks per scan stage
constexpr int kFChunkRows = 4 * kFChunkBlocks;          // kernel rows per stage (16 tiles of 8)
constexpr int kFStages = 3;                             // ring depth (scan and attention)
constexpr int kFMaxBpc = 192;                           // context blocks per CTA
constexpr int kFBmaxPitch = kFMaxBpc + 1;               // odd pitch: the 8 head rows of a warp hit 8 banks
constexpr int kFMaxCL = 16;
constexpr int kFListCap = 192;                          // block-list entries per CTA
constexpr int kFMaxKmax = 2048;                         // longest block list (kmax) the step takes

constexpr int cmax(int a, int b) { return a > b ? a : b; }
constexpr int round_up(int a, int m) { return (a + m - 1) / m * m; }

template <int D>
struct FLayout {
    // region A: scan ring | S, select scratch | attention ring | warp partials
    static constexpr int kChunkBytes = kFChunkRows * D * 2;
    static constexpr int kScanRing = kFStages * kChunkBytes;
    static constexpr int kBoxBytes = kBlock * 64 * 2;          // one TMA box: 64 keys x 64 dims
    static constexpr int kTileBytes = kBlock * D * 2;          // K or V of one block (D / 64 boxes)
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kAttnRing = kFStages * kStageBytes;
    static constexpr int kS = 0;                               // S of every block of the row
    static constexpr int kSelWs = kFMaxCL * kFMaxBpc * 4 + 16;  // bucket-select scratch (S may overhang 3)
    static constexpr int kSelEnd = kSelWs + (int)sizeof(CtaSelectSmem);
    static constexpr int kWo = 0;                              // [warp][16][kWoPitch] scaled warp outputs
    static constexpr int kWoPitch = D + 8;                     // floats; the 8 head rows a warp stores at once
                                                               // start 8 banks apart (conflict-free float2)
    static constexpr int kWml = kFWarps * 16 * kWoPitch * 4;   // [warp][16] m, then [warp][16] l
    static constexpr int kWf = kWml + 2 * kFWarps * 16 * 4;    // [warp][16] factors, [16] M, [16] L
    static constexpr int kMergeEnd = kWf + (kFWarps + 2) * 16 * 4;
    static constexpr int kRegionA = round_up(cmax(cmax(kScanRing, kAttnRing), cmax(kSelEnd, kMergeEnd)), 1024);
    // region B: block-maximum keys [16][kFBmaxPitch]; after the scores: combine slots and this CTA's list
    static constexpr int kBmax = kRegionA;
    static constexpr int kBmaxBytes = 16 * kFBmaxPitch * 4;
    static constexpr int kSlotPitch = D + 4;                   // floats: O[D], m, l (16-byte rows)
    static constexpr int kSlotBytes = 16 * kSlotPitch * 4;     // [heads / CL][CL][kSlotPitch]
    static constexpr int kMyList = kBmax + kSlotBytes;         // int32 [kFListCap] block ids
    static constexpr int kMyRows = kMyList + kFListCap * 4;    // int32 [kFListCap] first cache row of each
    static constexpr int kEnd = kBmax + cmax(kBmaxBytes, kSlotBytes + 2 * kFListCap * 4);
    static constexpr int kBytes = kEnd + 1024;                 // + slack to align the base to 1024 B
};

__device__ int g_fused_error = 0;
// testing only: when nonzero, the first kernel-cache wait of every CTA launched from now on gives up after this
// many polls (passed to the kernel as an argument, so the normal path reads nothing extra)
std::atomic<unsigned> g_first_wait_limit{0u};

// Bounded wait on a ring barrier: false after `limit` polls, or early once another thread of the CTA has marked a
// wait that ran out (checked every 256 polls, so a wait that succeeds within a few polls never reads it).
IV2_DEV bool fused_wait(uint64_t* bar, uint32_t parity, uint32_t limit, volatile int* cta_err)
{
    for (uint32_t i = 0; i < limit; ++i) {
        if (tc::mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u && *cta_err) return false;
    }
    *cta_err = 1;
    return false;
}

// order-preserving key -> float (inverse of float_key)
IV2_DEV float key_float(uint32_t k) { return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k); }

// q of one token, G heads as MMA rows, in the permuted head-dimension order of the scan (lane (gq, tq)
// holds d in [8 (4u + tq), +8) of rows gq and gq + 8), so a kernel row's 16-byte chunk is a B fragment
template <int D>
IV2_DEV void scan_q_permuted(const __nv_bfloat16* q_row0, int nrows, uint32_t (&qa)[D / 32][4],
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

IV2_DEV void online_merge(float& m, float& s, float m2, float s2)
{
    if (m2 == neg_inf()) return;
    if (m == neg_inf()) {
        m = m2;
        s = s2;
        return;
    }
    const float M = fmaxf(m, m2);
    s = s * ex2_approx(m - M) + s2 * ex2_approx(m2 - M);
    m = M;
}

// scores of one 8-kernel tile (rows j0t .. j0t + 7 of the stage; valid below `hi`) for rows gq, gq + 8
template <int D>
IV2_DEV void scan_tile(const unsigned char* rows, int row0, int nvalid, const uint32_t (&qa)[D / 32][4],
                       const uint32_t (&qb)[D / 32][4], float sl2, float (&z)[4])
{
    const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
    const bool ok = row0 + gq < nvalid;
    float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < D / 32; ++u) {
        uint4 kv = make_uint4(0, 0, 0, 0);
        if (ok) kv = *reinterpret_cast<const uint4*>(rows + (size_t)(row0 + gq) * D * 2 + (4 * u + tq) * 16);
        const uint32_t a0[4] = {qa[u][0], qb[u][0], qa[u][1], qb[u][1]};
        const uint32_t a1[4] = {qa[u][2], qb[u][2], qa[u][3], qb[u][3]};
        if (u & 1) {
            mma_bf16_16816(acc1, a0, kv.x, kv.y);
            mma_bf16_16816(acc1, a1, kv.z, kv.w);
        } else {
            mma_bf16_16816(acc0, a0, kv.x, kv.y);
            mma_bf16_16816(acc0, a1, kv.z, kv.w);
        }
    }
    const int ca = row0 + 2 * tq;
    const bool va = ca < nvalid, vb = ca + 1 < nvalid;
    z[0] = va ? (acc0[0] + acc1[0]) * sl2 : neg_inf();
    z[1] = vb ? (acc0[1] + acc1[1]) * sl2 : neg_inf();
    z[2] = va ? (acc0[2] + acc1[2]) * sl2 : neg_inf();
    z[3] = vb ? (acc0[3] + acc1[3]) * sl2 : neg_inf();
}

}  // namespace

template <int D, int CL, int E>
__global__ void __launch_bounds__(kFThreads, 2)
decode_fused_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                    QueryRows qr, __nv_bfloat16* __restrict__ kern, int nk_cap, MethodConsts mc, KvRows kr,
                    int32_t* __restrict__ idx, int32_t* __restrict__ cnt, __nv_bfloat16* __restrict__ out,
                    float* __restrict__ lse_out, unsigned first_wait_limit, const __nv_bfloat16* __restrict__ kraw,
                    int pool_new)
{
    using L = FLayout<D>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = tc::align_smem_1024(smem_raw);
    __shared__ uint64_t full[kFStages];
    __shared__ uint64_t never;  // testing only: a barrier no thread or copy arrives on
    __shared__ int cta_err;  // set by a wait that ran out: the CTA's other waits then give up early
    __shared__ __nv_bfloat16 new_kern[128];  // the kernel completed by the row's last key (pool_new)
    __shared__ float part_m[16], part_s[16], lse2[16], halo_out[16];
    __shared__ __align__(16) float lse_slot[kFMaxCL][16][2];  // (max, sum) partials pushed by every CTA

    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
    const int row = blockIdx.y;
    const int g = row % qr.Hkv, bt = row / qr.Hkv, t = bt % qr.T, b = bt / qr.T;
    const int G = qr.Hq / qr.Hkv;

    uint32_t* bmax = reinterpret_cast<uint32_t*>(smem + L::kBmax);
    if (tid < 16) {
        part_m[tid] = neg_inf();
        part_s[tid] = 0.f;
        halo_out[tid] = neg_inf();
    }
    for (int i = tid; i < 16 * kFBmaxPitch; i += kFThreads) bmax[i] = 0u;
    if (tid == 0) {
        for (int s = 0; s < kFStages; ++s) tc::mbar_init(&full[s], 1);
        tc::mbar_init(&never, 1);
        cta_err = 0;
        tc::fence_barrier_init();
        tc::prefetch_tensormap(&tmap_k);
        tc::prefetch_tensormap(&tmap_v);
    }
    __syncthreads();
    tc::cluster_arrive_release();  // block maxima zeroed: the CTA before may add its halo kernel from now on

    pdl_launch_dependents();
    pdl_wait();

    const int n = query_ctx(qr, b, t);
    const int c = (n - 1) / kBlock;
    const int nb = c + 1;
    // the draft model's sliding window (mc.window > 0): attend densely to the keys [w0, n), blocks bw .. c
    const int w0 = mc.window > 0 ? max(0, n - mc.window) : 0;
    const int bw = w0 / kBlock;
    const bool dense = mc.window > 0 || n <= mc.dense_len;
    const int nkv = min(num_kernels(n), nk_cap);
    const int bpc = ((nb + CL - 1) / CL + 3) & ~3;  // blocks per CTA, a multiple of 4
    const int b0 = rank * bpc, b1 = min(b0 + bpc, nb);
    const int nown = max(b1 - b0, 0);
    // a context past the launch's max_ctx would overrun the per-CTA tables: flag it, attend to nothing
    const bool bad = !dense && (bpc > kFMaxBpc || nb > kFThreads * E);
    // pool_new: the kernel completed by the row's last key (when it completes one) is pooled here by the CTA that
    // owns its block, with kernel_pool_kernel's arithmetic (two 16-key halves summed in row order in fp64, scaled
    // by 1/32, rounded once): its scan stage is patched with it and it is stored to the cache after the scan
    const int j_new = (pool_new && n >= kKernelSize && (n - kKernelSize) % kKernelStride == 0 && n <= qr.max_ctx)
                          ? (n - kKernelSize) / kKernelStride : -1;
    const bool own_new = j_new >= 0 && j_new < nk_cap && j_new / kKernelsPerBlock >= b0 &&
                         j_new / kKernelsPerBlock < b1;
    if (own_new && tid < D) {
        double half[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const long r0 = kv_pos_row(kr, b, (j_new + hh) * kKernelStride);  // 16 consecutive rows
            double acc = 0.0;
            if (r0 >= 0) {
                const __nv_bfloat16* src = kraw + (r0 * qr.Hkv + g) * D + tid;
#pragma unroll
                for (int r = 0; r < kKernelStride; ++r)
                    acc += (double)__bfloat162float(src[(size_t)r * qr.Hkv * D]);
            }
            half[hh] = acc;
        }
        const uint16_t bits = f64_to_bf16_rne((half[0] + half[1]) * (1.0 / kKernelSize));
        new_kern[tid] = *reinterpret_cast<const __nv_bfloat16*>(&bits);
    }
    const bool sparse = !dense && !bad;
    const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(qr.q) + ((size_t)bt * qr.Hq + g * G) * D;
    int32_t* idx_row = idx ? idx + (size_t)row * mc.kmax : nullptr;  // null: no block list is written
    const float sl2 = mc.scale * kLog2e;
    uint32_t phase_bits = 0;  // parity of each ring stage
    bool failed = bad;
    // A wait that runs out (bounded polls) marks the thread failed; the thread's later waits then give up after a
    // few polls, and every wait also gives up once another thread has marked the CTA (cta_err, checked every 256
    // polls, so a wait that succeeds on time never reads it).  Thread 0 issues every copy, and issues the copy
    // for ring position i + kFStages only while none of its own waits has run out: its own wait for position i
    // saw that buffer's copy land.  So after a failure the CTA issues no further copy; at its first wait that ran
    // out, thread 0 waits (bounded) for the copies of that ring it issued and did not see land, before the
    // stage barrier, so that no copy lands in region A once the loop is over.  The CTA still runs every loop (on
    // whatever the buffers hold: no address depends on the data) and takes part in every cluster barrier.  The
    // results of such a row are not the method's, and infllmv2_device_status reports the timeout.

    // ---------------- 1. scan this CTA's blocks of the kernel cache ----------------
    const int nch = (sparse && nown > 0) ? (nown + kFChunkBlocks - 1) / kFChunkBlocks : 0;
    if (nch > 0) {
        const __nv_bfloat16* kbase = kern + ((size_t)b * qr.Hkv + g) * nk_cap * D;
        auto issue_chunk = [&](int i) {
            const int sc = b0 + i * kFChunkBlocks, se = min(sc + kFChunkBlocks, b1);
            const int lo = sc * kKernelsPerBlock, hi = min(se * kKernelsPerBlock, nkv);
            uint64_t* bar = &full[i % kFStages];
            if (hi > lo) {
                tc::mbar_arrive_expect_tx(bar, (uint32_t)(hi - lo) * D * 2);
                tc::bulk_load(smem + (size_t)(i % kFStages) * L::kChunkBytes, kbase + (size_t)lo * D,
                              (uint32_t)(hi - lo) * D * 2, bar);
            } else {
                tc::mbar_arrive(bar);
            }
        };
        // the first stage goes out alone, ahead of the q load, so that its bytes are not queued behind the
        // other stages of every CTA of the launch; the rest of the ring follows once q is in registers
        if (tid == 0) issue_chunk(0);
        uint32_t qa[D / 32][4], qb[D / 32][4];
        scan_q_permuted<D>(qrow, G, qa, qb);
        if (tid == 0)
            for (int i = 1; i < kFStages && i < nch; ++i) issue_chunk(i);
        // running (max, sum) per row; the finite floor keeps 2^(m_old - m_new) free of inf - inf
        constexpr float kFloor = -1e30f;
        float lm[2] = {kFloor, kFloor}, ls[2] = {0.f, 0.f};
        const bool overlap = mc.membership == 0;
        const bool hv[2] = {gq < G, gq + 8 < G};

        for (int i = 0; i < nch; ++i) {
            const int st = i % kFStages;
            // testing only (a limit set from the host): the first wait polls a barrier nothing arrives on, so it
            // runs out after that many polls while the stage's copy is still in flight
            const bool test_wait = i == 0 && first_wait_limit != 0u;
            const bool landed = fused_wait(test_wait ? &never : &full[st], test_wait ? 0u : (phase_bits >> st) & 1u,
                                           test_wait ? first_wait_limit : failed ? 64u : (1u << 24), &cta_err);
            if (!landed) {
                if (tid == 0 && !failed)  // in flight: positions i .. i + kFStages - 1, each on its own stage
                    for (int j = i; j < nch && j < i + kFStages; ++j)
                        (void)tc::mbar_wait(&full[j % kFStages], (j / kFStages) & 1u, 1u << 20);
                failed = true;
            }
            phase_bits ^= 1u << st;
            const int sc = b0 + i * kFChunkBlocks, se = min(sc + kFChunkBlocks, b1);
            const int nblk = se - sc;
            if (own_new && j_new >= sc * kKernelsPerBlock && j_new < se * kKernelsPerBlock) {
                // the stage holds the cache's old row j_new: replace it with the pooled kernel
                __nv_bfloat16* prow = reinterpret_cast<__nv_bfloat16*>(smem + (size_t)st * L::kChunkBytes) +
                                      (size_t)(j_new - sc * kKernelsPerBlock) * D;
                if (tid < D) prow[tid] = new_kern[tid];
                tc::fence_proxy_async_smem();  // before the next copy into this stage
                __syncthreads();
            }
            const int nvalid = max(min(se * kKernelsPerBlock, nkv) - sc * kKernelsPerBlock, 0);  // rows staged
            const unsigned char* rows = smem + (size_t)st * L::kChunkBytes;
            // this warp's tiles: warp and warp + 8 of the stage's 16 (4 kernel rows per block, 8 per tile)
            float z[2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j) scan_tile<D>(rows, 8 * (warp + 8 * j), nvalid, qa, qb, sl2, z[j]);
            // LSE partials, branch-free (every row of the stage is owned by this CTA; invalid scores are -inf)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const float m4 = fmaxf(fmaxf(z[0][2 * r], z[0][2 * r + 1]), fmaxf(z[1][2 * r], z[1][2 * r + 1]));
                const float mn = fmaxf(lm[r], m4);
                ls[r] = ls[r] * ex2_approx(lm[r] - mn) + (ex2_approx(z[0][2 * r] - mn) + ex2_approx(z[0][2 * r + 1] - mn)) +
                        (ex2_approx(z[1][2 * r] - mn) + ex2_approx(z[1][2 * r + 1] - mn));
                lm[r] = mn;
            }
            // block maxima: tile j holds the stage's blocks 2 tt and 2 tt + 1 (tt = warp + 8 j) as cols 0..3 and
            // 4..7, so lane tq's two cols belong to block 2 tt + (tq >> 1).  Shuffle-free, one atomicMax per
            // lane for its own block; under the overlapping-window rule an odd lane's second col is the last
            // kernel of that block and also goes to the block after it (in this CTA, or the next CTA's first).
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int tt = warp + 8 * j;
                const int own = sc - b0 + 2 * tt + (tq >> 1);  // CTA-local block of this lane's cols
                const bool own_ok = 2 * tt + (tq >> 1) < nblk;
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const float v0 = z[j][2 * r], v1 = z[j][2 * r + 1];
                    // contained windows: a block's kernels are cols 0..2 of its four
                    const float vo = (!overlap && (tq & 1)) ? v0 : fmaxf(v0, v1);
                    uint32_t* bm = bmax + (gq + 8 * r) * kFBmaxPitch;
                    if (hv[r] && own_ok && vo != neg_inf()) atomicMax(&bm[own], float_key(vo));
                    if (overlap && (tq & 1) && hv[r] && own_ok && v1 != neg_inf()) {
                        if (own + 1 < nown) atomicMax(&bm[own + 1], float_key(v1));
                        else halo_out[gq + 8 * r] = v1;  // the CTA's last kernel: next CTA's block 0
                    }
                }
            }
            __syncthreads();  // stage consumed by every warp
            if (tid == 0 && !failed && i + kFStages < nch) issue_chunk(i + kFStages);
        }
        for (int r = 0; r < 2; ++r)
            if (lm[r] == kFloor) lm[r] = neg_inf();
        // per-head partials: the quad's lanes share rows gq, gq + 8; then the eight warps (region A is free)
        float* wred = reinterpret_cast<float*>(smem);  // [warp][16] max, then [warp][16] sum
#pragma unroll
        for (int r = 0; r < 2; ++r) {
#pragma unroll
            for (int o = 1; o <= 2; o <<= 1) {
                const float m2 = __shfl_xor_sync(0xffffffffu, lm[r], o);
                const float s2 = __shfl_xor_sync(0xffffffffu, ls[r], o);
                online_merge(lm[r], ls[r], m2, s2);
            }
            if (tq == 0) {
                wred[warp * 16 + gq + 8 * r] = lm[r];
                wred[kFWarps * 16 + warp * 16 + gq + 8 * r] = ls[r];
            }
        }
        __syncthreads();
        if (tid < 16) {
            float mw[kFWarps], m = neg_inf(), s = 0.f;
#pragma unroll
            for (int w = 0; w < kFWarps; ++w) {
                mw[w] = wred[w * 16 + tid];
                m = fmaxf(m, mw[w]);
            }
#pragma unroll
            for (int w = 0; w < kFWarps; ++w)
                s += (mw[w] == neg_inf()) ? 0.f : wred[kFWarps * 16 + w * 16 + tid] * ex2_approx(mw[w] - m);
            part_m[tid] = m;
            part_s[tid] = s;
        }
        __syncthreads();
    }
    tc::cluster_wait_acquire();  // every CTA's block maxima are initialised
    if (sparse) {
        // push the (max, sum) partials to every CTA, and the halo kernel to the next CTA's first block
        for (int item = tid; item < 8 * CL; item += kFThreads) {
            const int r = item / 8, h = 2 * (item % 8);
            *reinterpret_cast<float4*>(cluster.map_shared_rank(&lse_slot[0][0][0], r) + (rank * 16 + h) * 2) =
                make_float4(part_m[h], part_s[h], part_m[h + 1], part_s[h + 1]);
        }
        if (tid < G && rank + 1 < CL && b1 < nb && halo_out[tid] != neg_inf())
            atomicMax(cluster.map_shared_rank(bmax, rank + 1) + tid * kFBmaxPitch, float_key(halo_out[tid]));
    }
    cluster.sync();  // (A) partials and halo maxima in place; the scan rings are free

    // ---------------- 2. LSE and the group scores of this CTA's blocks, pushed to every CTA ----------------
    float* S = reinterpret_cast<float*>(smem + L::kS);
    if (sparse) {
        if (tid < G) {
            float mr[CL], m = neg_inf(), s = 0.f;
#pragma unroll
            for (int r = 0; r < CL; ++r) {
                mr[r] = lse_slot[r][tid][0];
                m = fmaxf(m, mr[r]);
            }
#pragma unroll
            for (int r = 0; r < CL; ++r) s += (mr[r] == neg_inf()) ? 0.f : lse_slot[r][tid][1] * ex2_approx(mr[r] - m);
            lse2[tid] = m == neg_inf() ? neg_inf() : m + __log2f(s);
        }
        __syncthreads();
        for (int k = tid; k < nown; k += kFThreads) {
            float acc = 0.f;
            const bool member = bmax[k] != 0u;
#pragma unroll
            for (int h = 0; h < 16; ++h) {
                const uint32_t key = bmax[h * kFBmaxPitch + k];
                if (h < G && key != 0u) acc += ex2_approx(key_float(key) - lse2[h]);
            }
            S[b0 + k] = member ? acc : neg_inf();
        }
        __syncthreads();
        // bpc is a multiple of 4, so b0 is 16-byte aligned; a tail past nb is never read
        const int nvec = (nown + 3) / 4;
        for (int item = tid; item < nvec * CL; item += kFThreads) {
            const int r = item % CL, v = item / CL;
            if (r != rank)
                *reinterpret_cast<float4*>(cluster.map_shared_rank(S, r) + b0 + 4 * v) =
                    *reinterpret_cast<const float4*>(S + b0 + 4 * v);
        }
    }
    cluster.sync();  // (B) every score of the row in every CTA

    // ---------------- 3. selection (every CTA, identical result; the leader writes it out) ----------------
    int32_t* my_list = reinterpret_cast<int32_t*>(smem + L::kMyList);
    // the first cache row of each of this CTA's blocks, found here by all threads (contiguous, packed or through
    // the page table) so that the thread issuing the copies only reads it; an unmapped page starts a block
    // before row 0, which the tensor map fills with zeros
    int32_t* my_row = reinterpret_cast<int32_t*>(smem + L::kMyRows);
    auto first_row = [&](int blk) {
        const long zr = kv_block_row(kr, b, blk);
        return zr >= 0 ? (int)zr : -kBlock;
    };
    int count = nb - bw;
    if (dense) {
        if (rank == 0 && tid < 32 && idx_row) warp_write_dense_row(c, mc.kmax, idx_row, cnt + row);
        for (int i = tid; rank + CL * i < count; i += kFThreads) my_row[i] = first_row(bw + rank + CL * i);
    } else if (bad) {
        count = 0;
        if (rank == 0 && tid == 0) cnt[row] = 0;
    } else {
        CtaSelectSmem& sel = *reinterpret_cast<CtaSelectSmem*>(smem + L::kSelWs);
        // this CTA's entries rank, rank + CL, ... straight from the select's emit (no pass over the whole list)
        const int total = cta_select_topk<kFThreads, E>(S, c, mc.init_blocks, mc.local_blocks, mc.topk, mc.kmax,
                                                        rank == 0 ? idx_row : nullptr, rank == 0 ? cnt + row : nullptr,
                                                        sel, [&](int pos, int blk) {
                                                            if (pos % CL == rank) {
                                                                my_list[pos / CL] = blk;
                                                                my_row[pos / CL] = first_row(blk);
                                                            }
                                                        });
        count = min(total, mc.kmax);
    }
    __syncthreads();
    // region A held generic-proxy data (scores, select scratch): order it before the TMA writes
    tc::fence_proxy_async_smem();

    // ---------------- 4. attention over this CTA's entries rank, rank + CL, ... ----------------
    const int my_n = count > rank ? (count - rank + CL - 1) / CL : 0;
    WarpAttnState<D> st;
    st.init();
    bool worked = false;
    {
        auto issue_block = [&](int i) {
            const int zrow = my_row[i];
            const int sidx = i % kFStages;
            unsigned char* stg = smem + (size_t)sidx * L::kStageBytes;
            tc::mbar_arrive_expect_tx(&full[sidx], (uint32_t)L::kStageBytes);
#pragma unroll
            for (int dh = 0; dh < D / 64; ++dh) {
                tc::tma_load_3d(stg + dh * L::kBoxBytes, &tmap_k, dh * 64, g, zrow, &full[sidx]);
                tc::tma_load_3d(stg + L::kTileBytes + dh * L::kBoxBytes, &tmap_v, dh * 64, g, zrow, &full[sidx]);
            }
        };
        if (tid == 0 && !failed)
            for (int i = 0; i < kFStages && i < my_n; ++i) issue_block(i);

        uint32_t qf[D / 16][4];
        load_q_rows<D>(qrow, G, qf);
        const int key0 = 8 * warp;           // this warp's keys of every block
        const int krow = key0 + (lane & 7);  // the key row this lane addresses in ldmatrix
        for (int i = 0; i < my_n; ++i) {
            const int sidx = i % kFStages;
            if (!fused_wait(&full[sidx], (phase_bits >> sidx) & 1u, failed ? 64u : (1u << 24), &cta_err)) {
                if (tid == 0 && !failed)  // as in the scan; a stage's parity also counts its uses by the scan
                    for (int j = i; j < my_n && j < i + kFStages; ++j) {
                        const int s = j % kFStages;
                        (void)tc::mbar_wait(&full[s], ((nch - s + kFStages - 1) / kFStages + j / kFStages) & 1u,
                                            1u << 20);
                    }
                failed = true;
            }
            phase_bits ^= 1u << sidx;
            const int blk = dense ? bw + rank + CL * i : my_list[i];
            const int nvalid = min(kBlock, n - blk * kBlock);
            const int nskip = max(0, w0 - blk * kBlock);  // keys of the block before the window (0 without one)
            unsigned char* stg = smem + (size_t)sidx * L::kStageBytes;
            // a warp works when one of its 8 keys is in [nskip, nvalid) (nskip < nvalid for every walked block),
            // so every row's running max is finite after its first block
            if (key0 < nvalid && key0 + 8 > nskip) {
                unsigned char* vt = stg + L::kTileBytes;
                if (key0 + 8 > nvalid) {
                    // rows past the context may hold anything: zero them so that 0 * V stays 0
                    for (int item = lane; item < 8 * (D / 8); item += 32) {
                        const int r = key0 + item / (D / 8), cidx = item % (D / 8);
                        if (r >= nvalid)
                            *reinterpret_cast<uint4*>(vt + (cidx >> 3) * L::kBoxBytes + r * 128 +
                                                      (((cidx & 7) ^ (r & 7)) << 4)) = make_uint4(0, 0, 0, 0);
                    }
                    tc::fence_proxy_async_smem();
                    __syncwarp();
                }
                // S = Q K^T over keys key0 .. key0 + 7
                float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < D / 32; ++kk) {
                    const int cidx = 4 * kk + (lane >> 3);
                    uint32_t b0r, b1r, b2r, b3r;
                    ldmatrix_x4(b0r, b1r, b2r, b3r,
                                stg + (cidx >> 3) * L::kBoxBytes + krow * 128 + (((cidx & 7) ^ (krow & 7)) << 4));
                    mma_bf16_16816(s4, qf[2 * kk], b0r, b1r);
                    mma_bf16_16816(s4, qf[2 * kk + 1], b2r, b3r);
                }
                const int ka = key0 + 2 * tq;
                const bool va = ka < nvalid && ka >= nskip, vb = ka + 1 < nvalid && ka + 1 >= nskip;
                float sc[4];
                sc[0] = va ? s4[0] * sl2 : neg_inf();
                sc[1] = vb ? s4[1] * sl2 : neg_inf();
                sc[2] = va ? s4[2] * sl2 : neg_inf();
                sc[3] = vb ? s4[3] * sl2 : neg_inf();
                float p[4];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    float mx = fmaxf(sc[2 * r], sc[2 * r + 1]);
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                    const float mnew = fmaxf(st.m[r], mx);
                    const float alpha = st.m[r] == neg_inf() ? 0.f : ex2_approx(st.m[r] - mnew);
                    st.m[r] = mnew;
                    st.l[r] *= alpha;
#pragma unroll
                    for (int nt = 0; nt < D / 8; ++nt) {
                        st.o[nt][2 * r] *= alpha;
                        st.o[nt][2 * r + 1] *= alpha;
                    }
                    p[2 * r] = ex2_approx(sc[2 * r] - mnew);
                    p[2 * r + 1] = ex2_approx(sc[2 * r + 1] - mnew);
                    st.l[r] += p[2 * r] + p[2 * r + 1];
                }
                const uint32_t pa0 = pack_bf16(p[0], p[1]), pa1 = pack_bf16(p[2], p[3]);
                // O += P V over the warp's 8 keys
#pragma unroll
                for (int nn = 0; nn < D / 32; ++nn) {
                    const int cidx = 4 * nn + (lane >> 3);
                    uint32_t v0r, v1r, v2r, v3r;
                    ldmatrix_x4_trans(v0r, v1r, v2r, v3r,
                                      vt + (cidx >> 3) * L::kBoxBytes + krow * 128 + (((cidx & 7) ^ (krow & 7)) << 4));
                    mma_bf16_1688(st.o[4 * nn + 0], pa0, pa1, v0r);
                    mma_bf16_1688(st.o[4 * nn + 1], pa0, pa1, v1r);
                    mma_bf16_1688(st.o[4 * nn + 2], pa0, pa1, v2r);
                    mma_bf16_1688(st.o[4 * nn + 3], pa0, pa1, v3r);
                }
                worked = true;
            }
            __syncthreads();  // stage consumed by every warp
            if (tid == 0 && !failed && i + kFStages < my_n) issue_block(i + kFStages);
        }
    }
    finalize_rows<D>(st);
    // the eight warp states -> this CTA's partial: factors 2^(m_w - M) once per (warp, head), then sums
    float* wo = reinterpret_cast<float*>(smem + L::kWo);  // [warp][16][kWoPitch]
    float* wm = reinterpret_cast<float*>(smem + L::kWml);  // [warp][16]
    float* wl = wm + kFWarps * 16;                         // [warp][16]
    float* wf = reinterpret_cast<float*>(smem + L::kWf);   // [warp][16]
    float* cM = wf + kFWarps * 16;                         // [16]
    float* cL = cM + 16;                                   // [16]
    if (tq == 0) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            wm[warp * 16 + gq + 8 * r] = worked ? st.m[r] : neg_inf();
            wl[warp * 16 + gq + 8 * r] = worked ? st.l[r] : 0.f;
        }
    }
    __syncthreads();
    if (tid < 16) {
        float M = neg_inf();
#pragma unroll
        for (int w = 0; w < kFWarps; ++w) M = fmaxf(M, wm[w * 16 + tid]);
        float Ls = 0.f;
#pragma unroll
        for (int w = 0; w < kFWarps; ++w) {
            const float mw = wm[w * 16 + tid];
            const float f = (mw == neg_inf()) ? 0.f : ex2_approx(mw - M);
            wf[w * 16 + tid] = f;
            Ls += f * wl[w * 16 + tid];
        }
        cM[tid] = M;
        cL[tid] = Ls;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int h = gq + 8 * r;
        const float f = wf[warp * 16 + h];
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt)
            *reinterpret_cast<float2*>(&wo[(warp * 16 + h) * L::kWoPitch + nt * 8 + 2 * tq]) =
                make_float2(st.o[nt][2 * r] * f, st.o[nt][2 * r + 1] * f);
    }
    __syncthreads();
    for (int item = tid; item < G * (D / 4); item += kFThreads) {
        const int h = item / (D / 4), d4 = (item % (D / 4)) * 4;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kFWarps; ++w) {
            const float4 v = *reinterpret_cast<const float4*>(&wo[(w * 16 + h) * L::kWoPitch + d4]);
            o.x += v.x;
            o.y += v.y;
            o.z += v.z;
            o.w += v.w;
        }
        float* slot = cluster.map_shared_rank(reinterpret_cast<float*>(smem + L::kBmax), h % CL) +
                      ((size_t)(h / CL) * CL + rank) * L::kSlotPitch;
        *reinterpret_cast<float4*>(slot + d4) = o;
        if (d4 == 0) *reinterpret_cast<float2*>(slot + D) = make_float2(cM[h], cL[h]);
    }
    cluster.sync();  // (C) every partial in its owner; no remote access after this

    // ---------------- 5. merge the CL partials of the heads this CTA owns ----------------
    const float* slots = reinterpret_cast<const float*>(smem + L::kBmax);
    for (int h = rank; h < G; h += CL) {
        const float* hs = slots + (size_t)(h / CL) * CL * L::kSlotPitch;
        for (int d = tid; d < D; d += kFThreads) {
            float M = neg_inf();
#pragma unroll
            for (int r = 0; r < CL; ++r) M = fmaxf(M, hs[r * L::kSlotPitch + D]);
            float O = 0.f, Lsum = 0.f;
            if (M != neg_inf()) {
#pragma unroll
                for (int r = 0; r < CL; ++r) {
                    const float mr = hs[r * L::kSlotPitch + D];
                    const float f = (mr == neg_inf()) ? 0.f : ex2_approx(mr - M);
                    O += hs[r * L::kSlotPitch + d] * f;
                    Lsum += hs[r * L::kSlotPitch + D + 1] * f;
                }
            }
            out[((size_t)bt * qr.Hq + g * G + h) * D + d] = __float2bfloat16_rn(Lsum > 0.f ? O / Lsum : 0.f);
            if (lse_out && d == 0)
                lse_out[(size_t)bt * qr.Hq + g * G + h] = Lsum > 0.f ? (M + __log2f(Lsum)) * kLn2 : neg_inf();
        }
    }
    // the pooled kernel goes to the cache (this CTA's copies of it have all landed; no other CTA reads it)
    if (own_new && tid < D) kern[(((size_t)b * qr.Hkv + g) * nk_cap + j_new) * D + tid] = new_kern[tid];
    // a wait that ran out (or a context past the launch's tables): the results of this row are not the method's
    if (failed) atomicOr(&g_fused_error, 1);
}

// ---------------------------------------------------------------- host
namespace {

template <int D, int CL, int E>
cudaError_t fused_launch(const CUtensorMap& tk, const CUtensorMap& tv, const QueryRows& qr, const void* kern,
                         int nk_cap, const MethodConsts& mc, const KvRows& kr, int32_t* idx, int32_t* cnt, void* out,
                         float* lse, const void* kraw, bool pool_new, cudaStream_t s)
{
    auto kfn = decode_fused_kernel<D, CL, E>;
    cudaError_t e = ensure_smem(kfn, FLayout<D>::kBytes);
    if (e != cudaSuccess) return e;
    if (CL > 8) {
        e = cudaFuncSetAttribute(kfn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    const int rows = qr.B * qr.T * qr.Hkv;
    return launch_pdl_cluster(kfn, dim3(CL, rows), dim3(kFThreads), CL, FLayout<D>::kBytes, s, tk, tv, qr,
                              static_cast<__nv_bfloat16*>(const_cast<void*>(kern)), nk_cap, mc, kr, idx, cnt,
                              static_cast<__nv_bfloat16*>(out), lse, g_first_wait_limit.load(std::memory_order_relaxed),
                              static_cast<const __nv_bfloat16*>(kraw), pool_new ? 1 : 0);
}

// 16-CTA clusters of this kernel the device keeps resident at once (0 when 16 is not schedulable).  Cached per
// device in an atomic (0: not yet known, else the count + 1), so that host threads calling at once are safe;
// two of them may both query the device, and store the same value.
template <int D, int E>
int resident_clusters16()
{
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    const int known = cached[dev].load(std::memory_order_relaxed);
    if (known > 0) return known - 1;
    int n = 0;
    auto kfn = decode_fused_kernel<D, 16, E>;
    if (ensure_smem(kfn, FLayout<D>::kBytes) == cudaSuccess &&
        cudaFuncSetAttribute(kfn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(16, 1);
        cfg.blockDim = dim3(kFThreads);
        cfg.dynamicSmemBytes = FLayout<D>::kBytes;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 16;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, kfn, &cfg) != cudaSuccess) n = 0;
    }
    (void)cudaGetLastError();
    cached[dev].store(n + 1, std::memory_order_relaxed);
    return n;
}

// 16-CTA clusters when every row fits in one wave of them (or the rows need 16), else 8-CTA clusters
template <int D, int E>
cudaError_t fused_dispatch_cl(const CUtensorMap& tk, const CUtensorMap& tv, const QueryRows& qr, const void* kern,
                              int nk_cap, const MethodConsts& mc, int nb_max, const KvRows& kr, int32_t* idx, int32_t* cnt,
                              void* out, float* lse, const void* kraw, bool pool_new, cudaStream_t s)
{
    const int rows = qr.B * qr.T * qr.Hkv;
    const bool need16 = nb_max > 8 * kFMaxBpc || mc.kmax > 8 * kFListCap;
    const int r16 = resident_clusters16<D, E>();
    if (need16 || (r16 > 0 && rows <= r16)) {
        if (r16 <= 0) return cudaErrorNotSupported;
        return fused_launch<D, 16, E>(tk, tv, qr, kern, nk_cap, mc, kr, idx, cnt, out, lse, kraw, pool_new, s);
    }
    return fused_launch<D, 8, E>(tk, tv, qr, kern, nk_cap, mc, kr, idx, cnt, out, lse, kraw, pool_new, s);
}

}  // namespace

bool decode_fused_supported(const QueryRows& qr, const MethodConsts& mc)
{
    const int nb_max = (qr.max_ctx - 1) / kBlock + 1;
    return nb_max <= kFMaxCL * kFMaxBpc && qr.Hq / qr.Hkv <= 16 && (qr.D == 64 || qr.D == 128) &&
           mc.kmax <= kFMaxKmax && mc.kmax <= kFMaxCL * kFListCap;
}

cudaError_t launch_decode_fused(const QueryRows& qr, const void* kern, int nk_cap, const MethodConsts& mc,
                                const void* k, const void* v, const KvRows& kr, int32_t* idx, int32_t* cnt, void* out,
                                float* lse, cudaStream_t s, bool pool_new)
{
    const int nb_max = (qr.max_ctx - 1) / kBlock + 1;
    if (!decode_fused_supported(qr, mc)) return cudaErrorNotSupported;
    CUtensorMap tk, tv;
    const uint64_t rowb = (uint64_t)qr.D * 2;
    // the rows the caches hold: every sequence's [0, Lcap), the packed rows, or the page pool
    if (!make_tma_map_bf16(&tk, k, qr.D, qr.Hkv, (uint64_t)kr.rows, rowb, rowb * qr.Hkv, 1, kBlock) ||
        !make_tma_map_bf16(&tv, v, qr.D, qr.Hkv, (uint64_t)kr.rows, rowb, rowb * qr.Hkv, 1, kBlock))
        return cudaErrorNotSupported;
    // the leader's top-k keeps E = ceil(nb_max / 256) blocks per thread
#define IV2_FUSED(DD, EE) \
    fused_dispatch_cl<DD, EE>(tk, tv, qr, kern, nk_cap, mc, nb_max, kr, idx, cnt, out, lse, k, pool_new, s)
    if (qr.D == 128) {
        if (nb_max <= 1024) return IV2_FUSED(128, 4);
        if (nb_max <= 2048) return IV2_FUSED(128, 8);
        return IV2_FUSED(128, 12);
    }
    if (nb_max <= 1024) return IV2_FUSED(64, 4);
    if (nb_max <= 2048) return IV2_FUSED(64, 8);
    return IV2_FUSED(64, 12);
#undef IV2_FUSED
}

// testing only: the poll limit of the first kernel-cache wait of every CTA (0: the normal wait)
int fused_set_first_wait_limit(unsigned polls)
{
    g_first_wait_limit.store(polls, std::memory_order_relaxed);
    return 0;
}

unsigned test_first_wait_limit() { return g_first_wait_limit.load(std::memory_order_relaxed); }

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

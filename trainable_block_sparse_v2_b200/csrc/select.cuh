// select.cuh -- top-k block selection with forced blocks, shared by the scoring kernels.
//
// Selection rule ("Tsinghua & ModelBest: MiniCPM4 technical details", "Model architecture: InfLLM v2",
// items 2-3; the workloads fix 1 initial and 2 local blocks): blocks [0, init) and [c - local + 1, c]
// are always kept; among the other blocks 0..c that have a visible kernel (S > -inf), the `topk` with
// the largest group score S are added, ties going to the lower block id.  The union is written in
// ascending order, padded with -1 up to kmax; the count goes to *cnt.
//
// Keys are the order-preserving uint32 image of S (non-candidates have key 0, below every float).  The
// k-th largest key is found by a bitwise search (one warp: 32 probes counted with warp reductions) or
// a radix select (whole CTA: 4 passes over 8-bit digits with shared-memory histograms).  Ties at the
// threshold are resolved by block id with a prefix count.
#pragma once

#include "common.cuh"

namespace iv2 {

IV2_DEV bool is_forced(int b, int c, int init, int local) { return b < init || (b > c - local && b <= c); }

// sum over the warp of a per-lane count in [0, 256): one ballot per bit, all independent
IV2_DEV int warp_count(int v)
{
    int total = 0;
#pragma unroll
    for (int bit = 0; bit < 8; ++bit) total += __popc(__ballot_sync(0xffffffffu, (v >> bit) & 1)) << bit;
    return total;
}

// ---------------------------------------------------------------------------------------------------
// one warp selects for one row; S in shared memory (nb = c + 1 entries, -inf = no visible kernel)
// ---------------------------------------------------------------------------------------------------
IV2_DEV void warp_select_topk(const float* S, int c, int init, int local, int topk, int kmax, int32_t* idx_out,
                              int32_t* cnt_out)
{
    const int lane = threadIdx.x & 31;
    const int nb = c + 1;
    auto key_of = [&](int b) -> uint32_t {
        const float s = S[b];
        return (!is_forced(b, c, init, local) && s != neg_inf()) ? float_key(s) : 0u;
    };
    int ncand = 0;
    for (int b = lane; b < nb; b += 32) ncand += key_of(b) != 0u;
    ncand = warp_count(ncand);

    uint32_t thr = 1u;  // keys >= thr are chosen (plus ties below)
    int need_eq = 0;    // how many keys == thr to take, lowest index first (only when thr is exact)
    bool all = ncand <= topk;
    if (!all) {
        uint32_t t = 0u;
        for (int bit = 31; bit >= 0; --bit) {
            const uint32_t probe = t | (1u << bit);
            int cntge = 0;
            for (int b = lane; b < nb; b += 32) cntge += key_of(b) >= probe;
            cntge = warp_count(cntge);
            if (cntge >= topk) t = probe;
        }
        // t is the k-th largest key
        int gt = 0;
        for (int b = lane; b < nb; b += 32) gt += key_of(b) > t;
        gt = warp_count(gt);
        thr = t;
        need_eq = topk - gt;
    }
    // emit ascending: chosen = forced || (key > thr) || (key == thr && rank among equals < need_eq)
    // (when all candidates are taken: key >= 1)
    int out_pos = 0, eq_seen = 0;
    for (int base = 0; base < nb; base += 32) {
        const int b = base + lane;
        const bool valid = b < nb;
        const bool forced = valid && is_forced(b, c, init, local);
        const uint32_t k = valid ? key_of(b) : 0u;
        bool chosen = forced || (all ? k != 0u : k > thr);
        if (!all) {
            const bool eq = valid && !forced && k == thr;
            const unsigned eqmask = __ballot_sync(0xffffffffu, eq);
            const int rank = eq_seen + __popc(eqmask & ((1u << lane) - 1u));
            if (eq && rank < need_eq) chosen = true;
            eq_seen += __popc(eqmask);
        }
        const unsigned cm = __ballot_sync(0xffffffffu, chosen);
        const int pos = out_pos + __popc(cm & ((1u << lane) - 1u));
        if (chosen && pos < kmax) idx_out[pos] = b;
        out_pos += __popc(cm);
    }
    for (int p = out_pos + lane; p < kmax; p += 32) idx_out[p] = -1;
    if (lane == 0) *cnt_out = out_pos;
}

// ---------------------------------------------------------------------------------------------------
// one warp selects for one row with a 256-bucket histogram in its own shared scratch; S in shared memory
// (nb = c + 1 <= 32 KW entries).  Lane l keeps blocks l, l + 32, ... in registers; the candidate keys are spread over
// the buckets by the same monotone fp32 map as the CTA select, the bucket B* holding the k-th largest key
// is found by a warp scan, and its members are ranked exactly by (key descending, block ascending).  The
// chosen set is identical to warp_select_topk's.
// ---------------------------------------------------------------------------------------------------
constexpr int kWarpBuckets = 256;
constexpr int kWarpMembers = 64;

struct WarpSelectSmem {
    int hist[kWarpBuckets];
    uint32_t mkey[kWarpMembers];
    int midx[kWarpMembers];
};

// KW = keys per lane kept in registers (nb <= 32 KW); lane l holds blocks l, l + 32, ...
template <int KW>
IV2_DEV void warp_select_topk_hist(const float* S, int c, int init, int local, int topk, int kmax, int32_t* idx_out,
                                   int32_t* cnt_out, WarpSelectSmem& ws)
{
    const int lane = threadIdx.x & 31;
    const int nb = c + 1;
    uint32_t key[KW];
    int ncand = 0;
    uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll
    for (int e = 0; e < KW; ++e) {
        const int b = lane + 32 * e;
        const float s = b < nb ? S[b] : neg_inf();
        key[e] = (b < nb && !is_forced(b, c, init, local) && s != neg_inf()) ? float_key(s) : 0u;
        if (key[e]) {
            ++ncand;
            lo = min(lo, key[e]);
            hi = max(hi, key[e]);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ncand += __shfl_xor_sync(0xffffffffu, ncand, o);
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    const bool all = ncand <= topk;
    const float bscale = hi > lo ? (float)(kWarpBuckets - 1) / (float)(hi - lo) : 0.f;
    int bk[KW];
    int bstar = kWarpBuckets;
    uint32_t tkey = 0u;
    int tidx = 0;
    if (!all) {
#pragma unroll
        for (int i = 0; i < kWarpBuckets / 32; ++i) ws.hist[lane + 32 * i] = 0;
        __syncwarp();
#pragma unroll
        for (int e = 0; e < KW; ++e) {
            bk[e] = key[e] ? min((int)((float)(key[e] - lo) * bscale), kWarpBuckets - 1) : -1;
            if (bk[e] >= 0) atomicAdd(&ws.hist[bk[e]], 1);
        }
        __syncwarp();
        // descending scan: lane l owns buckets [256 - 8 (l + 1), 256 - 8 l)
        constexpr int BPL = kWarpBuckets / 32;
        const int base = kWarpBuckets - BPL * (lane + 1);
        int cb[BPL], sum = 0;
#pragma unroll
        for (int j = 0; j < BPL; ++j) {
            cb[j] = ws.hist[base + BPL - 1 - j];  // descending within the lane
            sum += cb[j];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const int excl = incl - sum;
        int my_b = -1, my_above = 0, my_cnt = 0;
        if (excl < topk && topk <= incl) {
            int acc = excl;
#pragma unroll
            for (int j = 0; j < BPL; ++j) {
                if (my_b < 0 && acc + cb[j] >= topk) {
                    my_b = base + BPL - 1 - j;
                    my_above = acc;
                    my_cnt = cb[j];
                }
                acc += cb[j];
            }
        }
        const unsigned hitm = __ballot_sync(0xffffffffu, my_b >= 0);
        const int src = __ffs(hitm) - 1;
        bstar = __shfl_sync(0xffffffffu, my_b, src);
        const int rem = topk - __shfl_sync(0xffffffffu, my_above, src);  // members of B* still to take, >= 1
        const int bcnt = __shfl_sync(0xffffffffu, my_cnt, src);           // members of B*
        if (bcnt == rem) {
            // the boundary bucket is taken whole: every candidate in a bucket >= B* is chosen, no ranking
            tkey = 0u;
            tidx = 0x7fffffff;
        } else {
            // gather the members of B* (ascending block order) and count them
            int nm = 0;
#pragma unroll
            for (int e = 0; e < KW; ++e) {
                const bool mem = bk[e] == bstar;
                const unsigned mm = __ballot_sync(0xffffffffu, mem);
                const int pos = nm + __popc(mm & ((1u << lane) - 1u));
                if (mem && pos < kWarpMembers) {
                    ws.mkey[pos] = key[e];
                    ws.midx[pos] = lane + 32 * e;
                }
                nm += __popc(mm);
            }
            __syncwarp();
            if (nm <= kWarpMembers) {
                // the member of rank rem - 1 in (key descending, block ascending) order is the threshold
                int my_hit = -1;
                for (int i = lane; i < nm; i += 32) {
                    const uint32_t ki = ws.mkey[i];
                    const int ii = ws.midx[i];
                    int rank = 0;
                    for (int j = 0; j < nm; ++j) {
                        const uint32_t kj = ws.mkey[j];
                        rank += (kj > ki) || (kj == ki && ws.midx[j] < ii);
                    }
                    if (rank == rem - 1) my_hit = i;
                }
                const unsigned th = __ballot_sync(0xffffffffu, my_hit >= 0);
                const int ti = __shfl_sync(0xffffffffu, my_hit, __ffs(th) - 1);
                tkey = ws.mkey[ti];
                tidx = ws.midx[ti];
            } else {
                // many equal-bucket keys: bitwise search of the rem-th largest member key, then block ids
                uint32_t t = 0u;
                for (int bit = 31; bit >= 0; --bit) {
                    const uint32_t probe = t | (1u << bit);
                    int ge = 0;
#pragma unroll
                    for (int e = 0; e < KW; ++e) ge += bk[e] == bstar && key[e] >= probe;
                    if (warp_count(ge) >= rem) t = probe;
                }
                int gt = 0;
#pragma unroll
                for (int e = 0; e < KW; ++e) gt += bk[e] == bstar && key[e] > t;
                const int need = rem - warp_count(gt);
                // the need-th lowest block id among the members with key t
                int seen = 0;
                tidx = -1;
#pragma unroll
                for (int e = 0; e < KW; ++e) {
                    const unsigned eq = __ballot_sync(0xffffffffu, bk[e] == bstar && key[e] == t);
                    if (tidx < 0 && seen + __popc(eq) >= need) {
                        unsigned m2 = eq;
                        for (int j = 0; j < need - seen - 1; ++j) m2 &= m2 - 1u;
                        tidx = 32 * e + __ffs(m2) - 1;
                    }
                    seen += __popc(eq);
                }
                tkey = t;
            }
        }
        __syncwarp();
    }
    // emit ascending
    int out_pos = 0;
#pragma unroll
    for (int e = 0; e < KW; ++e) {
        const int b = lane + 32 * e;
        bool chosen = false;
        if (b < nb) {
            if (is_forced(b, c, init, local)) chosen = true;
            else if (key[e])
                chosen = all || bk[e] > bstar || (bk[e] == bstar && (key[e] > tkey || (key[e] == tkey && b <= tidx)));
        }
        const unsigned cm = __ballot_sync(0xffffffffu, chosen);
        const int pos = out_pos + __popc(cm & ((1u << lane) - 1u));
        if (chosen && pos < kmax) idx_out[pos] = b;
        out_pos += __popc(cm);
    }
    for (int p = out_pos + lane; p < kmax; p += 32) idx_out[p] = -1;
    if (lane == 0) *cnt_out = out_pos;
}

// dense row: every block 0..c, stored up to kmax entries, count c + 1
IV2_DEV void warp_write_dense_row(int c, int kmax, int32_t* idx_out, int32_t* cnt_out)
{
    const int lane = threadIdx.x & 31;
    for (int p = lane; p < kmax; p += 32) idx_out[p] = p <= c ? p : -1;
    if (lane == 0) *cnt_out = c + 1;
}

// ---------------------------------------------------------------------------------------------------
// the whole CTA (NT threads) selects for one row; S in shared memory
// ---------------------------------------------------------------------------------------------------
template <int NT>
IV2_DEV int cta_count(int local_count, int* red /* >= 2 * NT/32 ints */, int parity)
{
    const int w = threadIdx.x >> 5;
    local_count = __reduce_add_sync(0xffffffffu, local_count);
    int* slot = red + parity * (NT / 32);
    if ((threadIdx.x & 31) == 0) slot[w] = local_count;
    __syncthreads();
    int total = 0;
#pragma unroll
    for (int i = 0; i < NT / 32; ++i) total += slot[i];
    return total;
}

// exclusive prefix over threads (in thread order) of `v`; returns the prefix, *total gets the sum.  Threads may
// still read scan_smem when others return: the caller synchronises before scan_smem is written again.
template <int NT>
IV2_DEV int cta_exclusive_scan(int v, int* scan_smem /* NT/32 + 1 ints */, int* total)
{
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) scan_smem[w] = incl;
    __syncthreads();
    int wbase = 0, tot = 0;
#pragma unroll
    for (int i = 0; i < NT / 32; ++i) {
        const int s = scan_smem[i];
        if (i < w) wbase += s;
        tot += s;
    }
    *total = tot;
    return wbase + incl - v;
}

// E = max elements per thread (nb <= NT * E); thread tid owns blocks [tid*E, tid*E + E).
//
// Bucket select: the candidate keys are spread over kBuckets buckets by a monotone map of their value
// range, a shared histogram finds the bucket B* that holds the k-th largest key, and one warp ranks the
// few keys of B* exactly by (key descending, block ascending).  The rank-k element (T, I) of that total
// order is the threshold: a candidate is chosen iff (key, -block) >= (T, -I).  Counting uses no warp
// reductions in dependent loops (they are slow on sm_100): members are ranked by direct comparison.
constexpr int kBuckets = 2048;
constexpr int kMaxMembers = 1024;  // keys of the boundary bucket staged in shared memory
constexpr int kRankMembers = 128;  // up to this many are ranked by one warp; more: CTA-wide search

struct CtaSelectSmem {
    int hist[kBuckets];
    uint32_t mkey[kMaxMembers];
    int midx[kMaxMembers];
    int red[64];
    int nmem;
    uint32_t kmin, kmax;
    int bstar, above, bcount;  // boundary bucket, candidates in buckets above it, candidates in it
    uint32_t thr_key;
    int thr_idx;
};

// monotone (non-decreasing) map of a key in [kmin, kmax] to [0, kBuckets): every key goes through the
// same fp32 arithmetic, so equal keys share a bucket and a larger key never lands in a lower bucket
IV2_DEV int bucket_of(uint32_t key, uint32_t kmin, float bucket_scale)
{
    return min((int)((float)(key - kmin) * bucket_scale), kBuckets - 1);
}

// Returns the number of chosen blocks (every thread); on_entry(pos, block) is called, by the thread that owns
// the block, for every list entry pos < kmax; idx_out / cnt_out may be null (the list then only goes to on_entry).
struct NoListEntry {
    IV2_DEV void operator()(int, int) const {}
};

template <int NT, int E, typename OnEntry = NoListEntry>
IV2_DEV int cta_select_topk(const float* S, int c, int init, int local, int topk, int kmax, int32_t* idx_out,
                            int32_t* cnt_out, CtaSelectSmem& sm, OnEntry on_entry = OnEntry())
{
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nb = c + 1;
    const int b0 = threadIdx.x * E;
    uint32_t key[E];
    int ncand_local = 0;
    uint32_t lo = 0xffffffffu, hi = 0u;
    // the thread's E scores: with E a multiple of 4 and the whole range inside the row, E / 4 16-byte loads
    // (consecutive threads start 16 E bytes apart: no bank conflict, where E scalar loads conflict 4 ways)
    float sv[E];
    if constexpr (E % 4 == 0) {
        if (b0 + E <= nb) {
#pragma unroll
            for (int e4 = 0; e4 < E / 4; ++e4) {
                const float4 v = reinterpret_cast<const float4*>(S + b0)[e4];
                sv[4 * e4] = v.x;
                sv[4 * e4 + 1] = v.y;
                sv[4 * e4 + 2] = v.z;
                sv[4 * e4 + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e) sv[e] = b0 + e < nb ? S[b0 + e] : neg_inf();
        }
    } else {
#pragma unroll
        for (int e = 0; e < E; ++e) sv[e] = b0 + e < nb ? S[b0 + e] : neg_inf();
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int b = b0 + e;
        key[e] = 0u;
        if (b < nb && !is_forced(b, c, init, local)) {
            const float s = sv[e];
            if (s != neg_inf()) key[e] = float_key(s);
        }
        if (key[e] != 0u) {
            ++ncand_local;
            lo = min(lo, key[e]);
            hi = max(hi, key[e]);
        }
    }
    // candidate count and key range
    ncand_local = __reduce_add_sync(0xffffffffu, ncand_local);
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    if (lane == 0) {
        sm.red[warp] = ncand_local;
        sm.red[NW + warp] = (int)lo;
        sm.red[2 * NW + warp] = (int)hi;
    }
    for (int i = threadIdx.x; i < kBuckets; i += NT) sm.hist[i] = 0;
    if (threadIdx.x == 0) sm.nmem = 0;
    __syncthreads();
    int ncand = 0;
    uint32_t kmn = 0xffffffffu, kmx = 0u;
#pragma unroll
    for (int i = 0; i < NW; ++i) {
        ncand += sm.red[i];
        kmn = min(kmn, (uint32_t)sm.red[NW + i]);
        kmx = max(kmx, (uint32_t)sm.red[2 * NW + i]);
    }
    const bool all = ncand <= topk;
    const float bscale = kmx > kmn ? (float)(kBuckets - 1) / (float)(kmx - kmn) : 0.f;
    int bk[E];  // bucket of each key (unused for keys that are 0)
#pragma unroll
    for (int e = 0; e < E; ++e) bk[e] = bucket_of(key[e], kmn, bscale);
    int bstar = kBuckets;
    uint32_t tkey = 0u;
    int tidx = 0;
    if (!all) {
#pragma unroll
        for (int e = 0; e < E; ++e)
            if (key[e] != 0u) atomicAdd(&sm.hist[bk[e]], 1);
        __syncthreads();
        // descending suffix scan over buckets: thread t owns buckets [kBuckets - (t+1)*BPT, kBuckets - t*BPT)
        constexpr int BPT = kBuckets / NT;
        int cnt_b[BPT], sum = 0;
#pragma unroll
        for (int j = 0; j < BPT; ++j) {
            cnt_b[j] = sm.hist[kBuckets - 1 - (threadIdx.x * BPT + j)];
            sum += cnt_b[j];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        // red's last readers (the candidate count above) all passed the barrier after the histogram
        if (lane == 31) sm.red[warp] = incl;
        __syncthreads();
        int wbase = 0;
#pragma unroll
        for (int i = 0; i < NW; ++i)
            if (i < warp) wbase += sm.red[i];
        const int excl = wbase + incl - sum;  // candidates in buckets above this thread's range
        if (excl < topk && topk <= excl + sum) {
            int acc = excl;
#pragma unroll
            for (int j = 0; j < BPT; ++j) {
                if (acc + cnt_b[j] >= topk) {
                    sm.bstar = kBuckets - 1 - (threadIdx.x * BPT + j);
                    sm.above = acc;
                    sm.bcount = cnt_b[j];
                    break;
                }
                acc += cnt_b[j];
            }
        }
        __syncthreads();
        bstar = sm.bstar;
        const int rem = topk - sm.above;  // members of bucket B* still to take, >= 1
        if (sm.bcount == rem) {
            // the boundary bucket is taken whole (the usual case: its members are few): every candidate in a
            // bucket >= B* is chosen, with no ranking inside B* (the same for every thread: a uniform branch)
            tkey = 0u;
            tidx = 0x7fffffff;
        } else {
            // stage the members of B*
#pragma unroll
            for (int e = 0; e < E; ++e) {
                if (key[e] != 0u && bk[e] == bstar) {
                    const int slot = atomicAdd(&sm.nmem, 1);
                    if (slot < kMaxMembers) {
                        sm.mkey[slot] = key[e];
                        sm.midx[slot] = b0 + e;
                    }
                }
            }
            __syncthreads();
            if (sm.nmem > kRankMembers) {
                // degenerate spread (e.g. many equal scores): rank the bucket's members CTA-wide
                int parity = 0;
                uint32_t t = 0u;
                for (int bit = 31; bit >= 0; --bit) {
                    const uint32_t probe = t | (1u << bit);
                    int ge = 0;
#pragma unroll
                    for (int e = 0; e < E; ++e)
                        ge += key[e] != 0u && bk[e] == bstar && key[e] >= probe;
                    if (cta_count<NT>(ge, sm.red, parity) >= rem) t = probe;
                    parity ^= 1;
                }
                int gt = 0;
#pragma unroll
                for (int e = 0; e < E; ++e) gt += key[e] != 0u && bk[e] == bstar && key[e] > t;
                gt = cta_count<NT>(gt, sm.red, parity);
                parity ^= 1;
                const int need = rem - gt;
                int ti = 0;
                for (int bit = 12; bit >= 0; --bit) {
                    const int probe = ti | ((1 << bit) - 1);
                    int le = 0;
#pragma unroll
                    for (int e = 0; e < E; ++e) le += key[e] == t && (b0 + e) <= probe;
                    if (cta_count<NT>(le, sm.red, parity) < need) ti |= 1 << bit;
                    parity ^= 1;
                }
                if (threadIdx.x == 0) {
                    sm.thr_key = t;
                    sm.thr_idx = ti;
                }
            } else if (warp == 0) {
                // few members: the rank of member i in (key descending, block ascending) order is the number of
                // members before it; the one of rank rem-1 is the threshold
                const int nm = sm.nmem;
                for (int i = lane; i < nm; i += 32) {
                    const uint32_t ki = sm.mkey[i];
                    const int ii = sm.midx[i];
                    int rank = 0;
                    for (int j = 0; j < nm; ++j) {
                        const uint32_t kj = sm.mkey[j];
                        rank += (kj > ki) || (kj == ki && sm.midx[j] < ii);
                    }
                    if (rank == rem - 1) {
                        sm.thr_key = ki;
                        sm.thr_idx = ii;
                    }
                }
            }
            __syncthreads();
            tkey = sm.thr_key;
            tidx = sm.thr_idx;
        }
    }
    // emit ascending (branch-free: a key is 0 for blocks past nb, forced blocks and blocks with no kernel)
    bool chosen[E];
    int nchosen = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int b = b0 + e;
        const bool forced = b < nb && is_forced(b, c, init, local);
        const bool above =
            all || bk[e] > bstar || (bk[e] == bstar && (key[e] > tkey || (key[e] == tkey && b <= tidx)));
        chosen[e] = forced || (key[e] != 0u && above);
        nchosen += chosen[e];
    }
    int total;
    int pos = cta_exclusive_scan<NT>(nchosen, sm.red, &total);
#pragma unroll
    for (int e = 0; e < E; ++e) {
        if (chosen[e]) {
            if (pos < kmax) {
                if (idx_out) idx_out[pos] = b0 + e;
                on_entry(pos, b0 + e);
            }
            ++pos;
        }
    }
    if (idx_out)
        for (int p = total + threadIdx.x; p < kmax; p += NT) idx_out[p] = -1;
    if (cnt_out && threadIdx.x == 0) *cnt_out = total;
    return total;
}

}  // namespace iv2

// select.cuh -- top-k block selection with forced blocks, shared by the scoring kernels.
//
// Selection rule ("Tsinghua & ModelBest: MiniCPM4 technical details", "Model architecture: InfLLM v2",
// items 2-3; the workloads fix 1 initial and 2 local blocks): blocks [0, init) and [c - local + 1, c]
// are always kept; among the other blocks 0..c that have a visible kernel (S > -inf), the `topk` with
// the largest group score S are added, ties going to the lower block id.  The union is written in
// ascending order, padded with -1 up to kmax; the count goes to *cnt.
//
// The k-th largest key is found by a 32-step bitwise search on the order-preserving uint32 image of S
// (candidates only; non-candidates have key 0, below every float), counting keys >= the probe with
// warp reductions.  Ties at the threshold are resolved by index with a prefix count.
#pragma once

#include "common.cuh"

namespace iv2 {

IV2_DEV bool is_forced(int b, int c, int init, int local) { return b < init || (b > c - local && b <= c); }

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
    ncand = __reduce_add_sync(0xffffffffu, ncand);

    uint32_t thr = 1u;  // keys >= thr are chosen (plus ties below)
    int need_eq = 0;    // how many keys == thr to take, lowest index first (only when thr is exact)
    bool all = ncand <= topk;
    if (!all) {
        uint32_t t = 0u;
        for (int bit = 31; bit >= 0; --bit) {
            const uint32_t probe = t | (1u << bit);
            int cntge = 0;
            for (int b = lane; b < nb; b += 32) cntge += key_of(b) >= probe;
            cntge = __reduce_add_sync(0xffffffffu, cntge);
            if (cntge >= topk) t = probe;
        }
        // t is the k-th largest key
        int gt = 0;
        for (int b = lane; b < nb; b += 32) gt += key_of(b) > t;
        gt = __reduce_add_sync(0xffffffffu, gt);
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

// exclusive prefix over threads (in thread order) of `v`; returns the prefix, *total gets the sum
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
    __syncthreads();
    *total = tot;
    return wbase + incl - v;
}

// E = max elements per thread (nb <= NT * E); thread tid owns blocks [tid*E, tid*E + E)
template <int NT, int E>
IV2_DEV void cta_select_topk(const float* S, int c, int init, int local, int topk, int kmax, int32_t* idx_out,
                             int32_t* cnt_out, int* red /* >= 2*NT/32 + NT/32 + 1 ints */)
{
    const int nb = c + 1;
    const int b0 = threadIdx.x * E;
    uint32_t key[E];
    int ncand_local = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int b = b0 + e;
        key[e] = 0u;
        if (b < nb && !is_forced(b, c, init, local)) {
            const float s = S[b];
            if (s != neg_inf()) key[e] = float_key(s);
        }
        ncand_local += key[e] != 0u;
    }
    int* scan_smem = red + 2 * (NT / 32);
    int parity = 0;
    const int ncand = cta_count<NT>(ncand_local, red, parity);
    parity ^= 1;
    const bool all = ncand <= topk;
    uint32_t thr = 1u;
    int need_eq = 0;
    if (!all) {
        uint32_t t = 0u;
        for (int bit = 31; bit >= 0; --bit) {
            const uint32_t probe = t | (1u << bit);
            int ge = 0;
#pragma unroll
            for (int e = 0; e < E; ++e) ge += key[e] >= probe;
            const int tot = cta_count<NT>(ge, red, parity);
            parity ^= 1;
            if (tot >= topk) t = probe;
        }
        int gt = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) gt += key[e] > t;
        gt = cta_count<NT>(gt, red, parity);
        parity ^= 1;
        thr = t;
        need_eq = topk - gt;
    }
    // ties at the threshold: rank by block id
    int eq_local = 0;
    if (!all) {
#pragma unroll
        for (int e = 0; e < E; ++e) eq_local += key[e] == thr;
    }
    int eq_total;
    int eq_rank = cta_exclusive_scan<NT>(eq_local, scan_smem, &eq_total);
    bool chosen[E];
    int nchosen = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int b = b0 + e;
        bool ch = false;
        if (b < nb) {
            if (is_forced(b, c, init, local)) ch = true;
            else if (all) ch = key[e] != 0u;
            else if (key[e] > thr) ch = true;
            else if (key[e] == thr) {
                ch = eq_rank < need_eq;
                ++eq_rank;
            }
        }
        chosen[e] = ch;
        nchosen += ch;
    }
    int total;
    int pos = cta_exclusive_scan<NT>(nchosen, scan_smem, &total);
#pragma unroll
    for (int e = 0; e < E; ++e) {
        if (chosen[e]) {
            if (pos < kmax) idx_out[pos] = b0 + e;
            ++pos;
        }
    }
    for (int p = total + threadIdx.x; p < kmax; p += NT) idx_out[p] = -1;
    if (threadIdx.x == 0) *cnt_out = total;
}

}  // namespace iv2

// attn_warp.cuh -- warp-level block attention on mma.sync m16n8k16 (16 MMA rows = the G heads of one
// query token of a GQA group; 64-key blocks staged in swizzled shared memory; online softmax in log2 units).
#pragma once

#include "common.cuh"

namespace iv2 {

template <int D>
IV2_DEV uint32_t swz_kv(int r, int ch)
{
    return (uint32_t)(r * D * 2 + ((ch ^ (r & 7)) << 4));
}

template <int D>
struct KvTile {
    static constexpr int kBytes = kBlock * D * 2;  // one 64-key tile of K or V
};

// stage rows [0, 64) of a tile: row r comes from src + r * row_stride when r < nvalid, else zeros
template <int D>
IV2_DEV void warp_load_tile(unsigned char* dst, const __nv_bfloat16* src, size_t row_stride, int nvalid)
{
    constexpr int CH = D / 8;
    const int lane = threadIdx.x & 31;
#pragma unroll 4
    for (int i = lane; i < kBlock * CH; i += 32) {
        const int r = i / CH, ch = i % CH;
        const bool ok = r < nvalid;
        cp_async_16_zfill(dst + swz_kv<D>(r, ch), src + (ok ? (size_t)r * row_stride : 0) + ch * 8, ok ? 16 : 0);
    }
}

template <int D>
struct WarpAttnState {
    float o[D / 8][4];
    float m[2];  // running max, log2 units, rows gq and gq + 8
    float l[2];  // running sum (this lane's columns only until finalised)

    IV2_DEV void init()
    {
#pragma unroll
        for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
        m[0] = m[1] = neg_inf();
        l[0] = l[1] = 0.f;
    }
};

// q rows of one token: rows r < G are heads g*G + r; others zero.  Standard A-fragment layout.
template <int D>
IV2_DEV void load_q_rows(const __nv_bfloat16* q_row0, int G, uint32_t (&qf)[D / 16][4])
{
    const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = gq + 8 * (i & 1);
            const int dcol = ks * 16 + 2 * tq + 8 * (i >> 1);
            qf[ks][i] = r < G ? *reinterpret_cast<const uint32_t*>(q_row0 + (size_t)r * D + dcol) : 0u;
        }
}

// S = Q K^T for the staged K tile; acc[nt][4] = rows (gq, gq+8) x keys nt*8 + 2tq + {0,1}
template <int D>
IV2_DEV void tile_qk(const uint32_t (&qf)[D / 16][4], const unsigned char* ks_tile, float (&acc)[8][4])
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ks += 2) {
            const int r = nt * 8 + (lane & 7);
            const int ch = 2 * ks + (lane >> 3);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(b0, b1, b2, b3, ks_tile + swz_kv<D>(r, ch));
            mma_bf16_16816(acc[nt], qf[ks], b0, b1);
            mma_bf16_16816(acc[nt], qf[ks + 1], b2, b3);
        }
    }
}

// online softmax update with the scores of one tile (already scaled to log2 units and masked),
// then O += P V with the staged V tile
template <int D>
IV2_DEV void tile_softmax_pv(WarpAttnState<D>& st, float (&s)[8][4], const unsigned char* vs_tile)
{
    const int lane = threadIdx.x & 31;
    float mnew[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        float mx = st.m[i];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * i], s[nt][2 * i + 1]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        mnew[i] = mx;
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float ref = mnew[i] == neg_inf() ? 0.f : mnew[i];
        const float alpha = exp2_fast(st.m[i] - ref);  // 0 when the old max is -inf
        st.l[i] *= alpha;
#pragma unroll
        for (int nd = 0; nd < D / 8; ++nd) {
            st.o[nd][2 * i] *= alpha;
            st.o[nd][2 * i + 1] *= alpha;
        }
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            s[nt][2 * i] = exp2_fast(s[nt][2 * i] - ref);
            s[nt][2 * i + 1] = exp2_fast(s[nt][2 * i + 1] - ref);
            st.l[i] += s[nt][2 * i] + s[nt][2 * i + 1];
        }
        st.m[i] = mnew[i];
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {  // 16 keys per k-step
        uint32_t a[4];
        a[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
        a[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
        a[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        a[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
        for (int nd = 0; nd < D / 8; nd += 2) {
            const int mi = lane >> 3;
            const int r = 16 * kk + (mi & 1) * 8 + (lane & 7);
            const int ch = nd + (mi >> 1);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4_trans(b0, b1, b2, b3, vs_tile + swz_kv<D>(r, ch));
            mma_bf16_16816(st.o[nd], a, b0, b1);
            mma_bf16_16816(st.o[nd + 1], a, b2, b3);
        }
    }
}

// scale to log2 units and mask: key column c valid iff (valid_mask >> c) & 1 (64-bit mask)
IV2_DEV void scale_mask(float (&acc)[8][4], float sl2, uint64_t valid)
{
    const int tq = threadIdx.x & 3;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int col = nt * 8 + 2 * tq + e;
            const bool ok = (valid >> col) & 1ull;
            acc[nt][e] = ok ? acc[nt][e] * sl2 : neg_inf();
            acc[nt][2 + e] = ok ? acc[nt][2 + e] * sl2 : neg_inf();
        }
}

IV2_DEV uint64_t prefix_mask64(int nvalid)
{
    return nvalid >= 64 ? ~0ull : (nvalid <= 0 ? 0ull : ((1ull << nvalid) - 1ull));
}

// the k-th block of a row's list; -1 when absent or invalid
IV2_DEV int row_block(bool dense, int c, const int32_t* idx_row, int count, int k, int n)
{
    if (dense) return k <= c ? k : -1;
    if (k >= count) return -1;
    const int blk = idx_row[k];
    return (blk >= 0 && blk * kBlock < n) ? blk : -1;
}

// finalise the row sums across the 4 lanes of a row
template <int D>
IV2_DEV void finalize_rows(WarpAttnState<D>& st)
{
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        st.l[i] += __shfl_xor_sync(0xffffffffu, st.l[i], 1);
        st.l[i] += __shfl_xor_sync(0xffffffffu, st.l[i], 2);
    }
}

}  // namespace iv2

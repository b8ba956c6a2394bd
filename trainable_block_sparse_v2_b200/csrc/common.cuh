// common.cuh -- device helpers shared by the InfLLM v2 kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define IV2_DEV __device__ __forceinline__

namespace iv2 {

// ---- method geometry supported by the GPU kernels ------------------------------------------------
constexpr int kBlock = 64;          // keys per context block
constexpr int kKernelSize = 32;     // keys per semantic-kernel window
constexpr int kKernelStride = 16;   // window stride
constexpr int kKernelsPerBlock = kBlock / kKernelStride;  // 4 window starts per block

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

IV2_DEV float neg_inf() { return __int_as_float(0xff800000); }

// number of complete kernel windows over the first n keys
IV2_DEV int num_kernels(int n) { return n >= kKernelSize ? (n - kKernelSize) / kKernelStride + 1 : 0; }

// kernels of block `blk` under the membership rule (0 = OVERLAP: windows intersecting the block,
// 1 = CONTAINED: windows inside it), as the half-open range [lo, hi) before clipping to visibility
IV2_DEV void block_kernel_range(int blk, int membership, int& lo, int& hi)
{
    if (membership == 0) {
        lo = blk * kKernelsPerBlock - (kKernelSize / kKernelStride - 1);
        hi = blk * kKernelsPerBlock + kKernelsPerBlock;
    } else {
        lo = blk * kKernelsPerBlock;
        hi = blk * kKernelsPerBlock + kKernelsPerBlock - (kKernelSize / kKernelStride - 1);
    }
}

// ---- bf16 packing --------------------------------------------------------------------------------
IV2_DEV uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// fp64 -> bf16, round to nearest even, in one correctly rounded step: round to odd into fp32 first (fp32 has
// at least two more significand bits than bf16, so the second rounding equals a direct one; Boldo and
// Melquiond, IEEE Trans. Computers 57(4), 2008).  The semantic kernels are rounded through it.
IV2_DEV uint16_t f64_to_bf16_rne(double x)
{
    float f = __double2float_rz(x);                 // truncate toward zero into fp32
    if ((double)f != x) f = __uint_as_float(__float_as_uint(f) | 1u);  // inexact: make the last bit odd
    __nv_bfloat16 h = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&h);
}

IV2_DEV float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
IV2_DEV float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// ---- legacy tensor-core MMA: D[16x8] += A[16x16] * B[16x8], bf16 in, fp32 accumulate -------------
// Fragment layout (lane = 4*g + t): A regs {a0: (g, 2t..2t+1), a1: (g+8, 2t..), a2: (g, 2t+8..), a3: (g+8, 2t+8..)},
// B regs {b0: (k 2t..2t+1, n g), b1: (k 2t+8.., n g)}, C regs {c0,c1: (g, 2t..2t+1), c2,c3: (g+8, 2t..)}.
IV2_DEV void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D (+)= A * B, m16n8k8, bf16 in, f32 accumulate; a0 = (row g, cols 2t..2t+1), a1 = (row g+8, ...),
// b0 = (k 2t..2t+1, n g)
IV2_DEV void mma_bf16_1688(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t b0)
{
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};\n"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a0), "r"(a1), "r"(b0));
}

IV2_DEV void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, const void* smem_row_ptr)
{
    uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(smem_row_ptr));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(a));
}

IV2_DEV void ldmatrix_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, const void* smem_row_ptr)
{
    uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(smem_row_ptr));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(a));
}

// ---- asynchronous global -> shared copies --------------------------------------------------------
IV2_DEV void cp_async_16(void* smem, const void* gmem)
{
    uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}

// zero-fill variant: copies `src_bytes` (0 or 16) and fills the rest of the 16 bytes with zeros
IV2_DEV void cp_async_16_zfill(void* smem, const void* gmem, int src_bytes)
{
    uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(src_bytes));
}

IV2_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }

template <int N>
IV2_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// ---- streaming loads -----------------------------------------------------------------------------
IV2_DEV uint4 ld_nc_v4(const void* p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// ---- order-preserving float -> uint32 (larger float -> larger key; 0 is below every float) -------
IV2_DEV uint32_t float_key(float f)
{
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---- warp reductions -----------------------------------------------------------------------------
IV2_DEV float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

IV2_DEV float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ---- programmatic dependent launch ---------------------------------------------------------------
// Every kernel lets the next kernel of the stream start launching at once, and waits for the previous
// kernel of the stream to finish (and its writes to be visible) before touching global memory.  The
// wait is the hardware's grid dependency, not a spin loop.
IV2_DEV void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
IV2_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// fast 2^x (MUFU) -- inputs are <= 0 or -inf on every use in this library
IV2_DEV float exp2_fast(float x) { return exp2f(x); }

// the hardware 2^x approximation (MUFU.EX2, flush-to-zero): 2^-inf = 0; used where the result is rounded
// to bf16 right away
IV2_DEV float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

}  // namespace iv2

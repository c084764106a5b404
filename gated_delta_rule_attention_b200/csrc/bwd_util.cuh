// bwd_util.cuh -- register-tiled products on shared-memory operands, shared by the
// backward kernels.
#pragma once

#include <cstdint>

namespace la {

// Register-tiled products on shared-memory operands.  A thread computes RM rows x RN
// columns of an M x N output: rows r0 + i (i < RM) and columns lane + 32 n (n < RN), so
// that the B operand's loads are consecutive across the warp and the A operand's are
// broadcasts.  acc[i][n] += sum_k A(row, k) B(k, col).
template <int RM, int RN, int K, typename FA, typename FB>
__device__ __forceinline__ void tile_mma(float (&acc)[RM][RN], int r0, int lane, FA a, FB b) {
#pragma unroll 4
    for (int kk = 0; kk < K; ++kk) {
        float av[RM], bv[RN];
#pragma unroll
        for (int i = 0; i < RM; ++i) av[i] = a(r0 + i, kk);
#pragma unroll
        for (int n = 0; n < RN; ++n) bv[n] = b(kk, lane + 32 * n);
#pragma unroll
        for (int i = 0; i < RM; ++i)
#pragma unroll
            for (int n = 0; n < RN; ++n) acc[i][n] = fmaf(av[i], bv[n], acc[i][n]);
    }
}

// Warp-level products on the tensor cores (mma.sync m16n8k8, tf32 operands, fp32
// accumulate): d[nt] += sum_{k<K} A(m, k) B(k, n) for the 16 x 8 NT block at rows m0..m0+15,
// columns n0..n0+8 NT-1.  The accessors return fp32; with SPLIT each operand is split into
// a tf32 high part and a tf32 remainder and three products keep fp32 accuracy
// (hi*hi + hi*lo + lo*hi), else the operands are rounded to tf32 once.
// Element r of d[nt] sits at row m0 + (lane >> 2) + 8 (r >> 1), column
// n0 + 8 nt + 2 (lane & 3) + (r & 1).
__device__ __forceinline__ uint32_t tf32_bits(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void mma_16x8x8_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                                uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
template <int NT, int K, bool SPLIT, typename FA, typename FB>
__device__ __forceinline__ void warp_mma(float (&d)[NT][4], int m0, int n0, FA a, FB b) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
#pragma unroll 2
    for (int kk = 0; kk < K; kk += 8) {
        const float af[4] = {a(m0 + g, kk + t4), a(m0 + g + 8, kk + t4), a(m0 + g, kk + t4 + 4),
                             a(m0 + g + 8, kk + t4 + 4)};
        uint32_t ah[4], al[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            ah[i] = tf32_bits(af[i]);
            if (SPLIT) al[i] = tf32_bits(af[i] - __uint_as_float(ah[i]));
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float b0 = b(kk + t4, n0 + 8 * nt + g), b1 = b(kk + t4 + 4, n0 + 8 * nt + g);
            const uint32_t bh0 = tf32_bits(b0), bh1 = tf32_bits(b1);
            mma_16x8x8_tf32(d[nt], ah, bh0, bh1);
            if (SPLIT) {
                mma_16x8x8_tf32(d[nt], ah, tf32_bits(b0 - __uint_as_float(bh0)),
                                tf32_bits(b1 - __uint_as_float(bh1)));
                mma_16x8x8_tf32(d[nt], al, bh0, bh1);
            }
        }
    }
}

}  // namespace la

// bwd_util.cuh -- register-tiled products on shared-memory operands, shared by the
// backward kernels.
#pragma once

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

}  // namespace la

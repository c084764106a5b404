// bwd_util.cuh -- products on shared-memory operands (register-tiled CUDA-core and
// warp-level tensor-core forms), cp.async staging and reductions shared by the backward
// kernels.  Include after la_internal.cuh (to_f32).
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
// columns n0..n0+8 NT-1.  The accessors return fp32.  An operand marked for splitting is
// taken as a tf32 high part plus a tf32 remainder, and the products keep fp32 accuracy
// (hi*hi + hi*lo + lo*hi); an unsplit operand is rounded to tf32 once, which is exact for
// values that came from bf16.
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
template <int NT, int K, bool SPLIT, bool SPLIT_B = SPLIT, typename FA, typename FB>
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
            if (SPLIT_B)
                mma_16x8x8_tf32(d[nt], ah, tf32_bits(b0 - __uint_as_float(bh0)),
                                tf32_bits(b1 - __uint_as_float(bh1)));
            if (SPLIT) mma_16x8x8_tf32(d[nt], al, bh0, bh1);
        }
    }
}

// Warp-level bf16 products (mma.sync m16n8k16, fp32 accumulate): d += A B for one 16 x 8
// block; element r of d sits as in warp_mma.  The fragments come from ldmatrix below.
__device__ __forceinline__ void mma_16x8x16_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                                 uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// ---- bf16 fragments by ldmatrix for mma.sync m16n8k16 (tiles row-major in shared memory,
// pitch in bf16 elements; 16-byte aligned rows; a pitch of 2P bytes = 16 (mod 32) avoids
// bank conflicts)
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_addr(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_addr(p)));
}
__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1]) : "r"(smem_addr(p)));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t (&r)[2], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1]) : "r"(smem_addr(p)));
}
// The A fragment (rows m0..m0+15, k0..k0+15) of A = X (X row-major [m][k]) or, with TRANS,
// of A = X^T (X row-major [k][m]).
template <bool TRANS>
__device__ __forceinline__ void frag_a(uint32_t (&a)[4], const __nv_bfloat16 *X, int pitch, int m0, int k0) {
    const int l = threadIdx.x & 31;
    if (!TRANS) ldsm_x4(a, X + (m0 + (l & 15)) * pitch + k0 + 8 * (l >> 4));
    else ldsm_x4_t(a, X + (k0 + (l & 7) + 8 * (l >> 4)) * pitch + m0 + 8 * ((l >> 3) & 1));
}
// The B fragment (k0..k0+15, n0..n0+7) of B = X^T (X row-major [n][k]) or, with TRANS, of
// B = X (X row-major [k][n]).
template <bool TRANS>
__device__ __forceinline__ void frag_b(uint32_t (&b)[2], const __nv_bfloat16 *X, int pitch, int k0, int n0) {
    const int l = threadIdx.x & 15;
    if (!TRANS) ldsm_x2(b, X + (n0 + (l & 7)) * pitch + k0 + 8 * (l >> 3));
    else ldsm_x2_t(b, X + (k0 + l) * pitch + n0);
}
// frag_a<false> on a 128B-swizzled tile of 64-element rows (chunk j of row r at chunk
// j ^ (r & 7), no padding): the A fragment (rows m0..m0+15, k0..k0+15).
__device__ __forceinline__ void frag_a_sw64(uint32_t (&a)[4], const __nv_bfloat16 *X, int m0, int k0) {
    const int l = threadIdx.x & 31;
    const int r = m0 + (l & 15), j = (k0 >> 3) + (l >> 4);
    ldsm_x4(a, X + r * 64 + 8 * (j ^ (r & 7)));
}
// frag_b on an unpadded tile of rows of `w` elements (w >= 64) whose 16-byte chunks are
// XOR-swizzled by the row: chunk j of row r sits at chunk j ^ (r & 7).  Eight consecutive
// rows at one logical chunk then fall in eight different bank groups.
template <bool TRANS>
__device__ __forceinline__ void frag_b_sw(uint32_t (&b)[2], const __nv_bfloat16 *X, int w, int k0, int n0) {
    const int l = threadIdx.x & 15;
    if (!TRANS) {
        const int r = n0 + (l & 7), j = (k0 >> 3) + (l >> 3);
        ldsm_x2(b, X + r * w + 8 * (j ^ (r & 7)));
    } else {
        const int r = k0 + l;
        ldsm_x2_t(b, X + r * w + 8 * ((n0 >> 3) ^ (r & 7)));
    }
}
// d[nt] += A B over K for the 16 x 8 NT block at (m0, n0), A and B bf16 tiles; an operand
// given with a second (remainder) tile is taken as high + low parts: products
// hi*hi + hi*lo + lo*hi (a computed fp32 value v = bf16(v) + bf16(v - bf16(v)) to 2^-17).
// With SWB, B is a swizzled tile (frag_b_sw) and pb its row length.
template <int NT, int K, bool TA, bool TB, bool SWB = false>
__device__ __forceinline__ void mma_bf16_tiles(float (&d)[NT][4], int m0, int n0,
                                               const __nv_bfloat16 *A, const __nv_bfloat16 *Alo, int pa,
                                               const __nv_bfloat16 *B, const __nv_bfloat16 *Blo, int pb) {
    auto fb = [&](uint32_t (&b)[2], const __nv_bfloat16 *X, int kk, int n) {
        if constexpr (SWB) frag_b_sw<TB>(b, X, pb, kk, n);
        else frag_b<TB>(b, X, pb, kk, n);
    };
#pragma unroll
    for (int kk = 0; kk < K; kk += 16) {
        uint32_t a[4], al[4];
        frag_a<TA>(a, A, pa, m0, kk);
        if (Alo) frag_a<TA>(al, Alo, pa, m0, kk);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            uint32_t b[2];
            fb(b, B, kk, n0 + 8 * nt);
            mma_16x8x16_bf16(d[nt], a, b[0], b[1]);
            if (Blo) {
                uint32_t bl[2];
                fb(bl, Blo, kk, n0 + 8 * nt);
                mma_16x8x16_bf16(d[nt], a, bl[0], bl[1]);
            }
            if (Alo) mma_16x8x16_bf16(d[nt], al, b[0], b[1]);
        }
    }
}
// v as bf16 high and low parts
__device__ __forceinline__ void split_bf16(float v, __nv_bfloat16 &hi, __nv_bfloat16 &lo) {
    hi = __float2bfloat16_rn(v);
    lo = __float2bfloat16_rn(v - __bfloat162float(hi));
}

// ---- cp.async staging of raw inputs (16-byte copies into shared memory)
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Rows [0, n) of `w` elements (w * sizeof(IO) a multiple of 16 bytes) from src (row stride
// ld elements, 16-byte aligned rows) into dst (row stride w); NT threads take part.
template <int NT, typename IO>
__device__ __forceinline__ void stage_rows(void *dst, const IO *src, int ld, int w, int n) {
    constexpr int E = 16 / sizeof(IO);   // elements per copy
    const int per = w / E;
    for (int p = threadIdx.x; p < n * per; p += NT) {
        const int t = p / per, x = (p % per) * E;
        cp_async16(static_cast<IO *>(dst) + t * w + x, src + (size_t)t * ld + x);
    }
}
// `rows` staged rows of w elements into an fp32 tile (pitch a multiple of 4 floats), zero
// past row n: 16 bytes of staged elements per step, written as float4.
template <int NT, typename IO>
__device__ __forceinline__ void unstage(const void *src, int rows, int w, int n, float *dst, int pitch) {
    constexpr int E = 16 / sizeof(IO);
    for (int p = threadIdx.x; p < rows * w / E; p += NT) {
        const int t = p * E / w, j = p * E % w;
        float f[E];
        if (t < n) {
            const uint4 raw = *reinterpret_cast<const uint4 *>(static_cast<const IO *>(src) + t * w + j);
            const IO *x = reinterpret_cast<const IO *>(&raw);
#pragma unroll
            for (int e = 0; e < E; ++e) f[e] = to_f32(x[e]);
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e) f[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < E; e += 4)
            *reinterpret_cast<float4 *>(dst + t * pitch + j + e) = make_float4(f[e], f[e + 1], f[e + 2], f[e + 3]);
    }
}
// p[0] += a, p[1] += b in global memory (one vector reduction; p 8-byte aligned).
__device__ __forceinline__ void red_add2(float *p, float a, float b) {
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(a), "f"(b) : "memory");
}

}  // namespace la

// tc_util.cuh -- device helpers shared by the tensor-core prefill kernels: operand
// descriptors, K-step MMA chains, fast exp2/log2, bf16 tile stores and scaling, and the
// 64x64 unit lower-triangular inverse of the delta-rule chunk (warp-level tf32 products).
#pragma once

#include "ptx.cuh"

namespace la {
namespace tc {

using namespace ptx;

// Row stride (floats) of the fp32 64x64 scratch matrices of the triangular inverse.
constexpr uint32_t kLmStride = 65;

__device__ __forceinline__ uint64_t dk(uint32_t addr) { return sdesc_sw128(addr, 16, 1024); }
__device__ __forceinline__ uint64_t dmn(uint32_t addr, uint32_t lbo) {
    return sdesc_sw128(addr, lbo, 1024);
}

// D (+)= A B over NK steps of K = 16, issued back to back.  The operand descriptors are
// built once; each step adds its offset to the start-address field (16-byte units), a
// compile-time constant once the loop is unrolled.  A K-major 128B-swizzled operand
// advances 32 bytes per step inside a 64-column half and jumps to the next half
// (KHALF bytes further) every four steps; an MN-major one advances 8 K rows = 2048 bytes.
template <int NK, bool A_KMAJ, bool B_KMAJ, uint32_t A_KHALF = 16384, uint32_t B_KHALF = 16384>
__device__ __forceinline__ void mma_chain(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, bool accumulate_first) {
#pragma unroll
    for (int ks = 0; ks < NK; ++ks) {
        const uint64_t ao = A_KMAJ ? (((ks >> 2) * A_KHALF + (ks & 3) * 32) >> 4) : (uint64_t)(ks * 128);
        const uint64_t bo = B_KMAJ ? (((ks >> 2) * B_KHALF + (ks & 3) * 32) >> 4) : (uint64_t)(ks * 128);
        mma_bf16_ss(d_tmem, a_desc + ao, b_desc + bo, idesc, accumulate_first || ks > 0);
    }
}
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Bounded wait that ignores the abort flag (used to drain in-flight work on exit).
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
#pragma unroll 1
    for (uint32_t i = 0; i < kSpinLimit; ++i)
        if (mbar_try_wait(bar, parity)) return;
}

// Write 16 fp32 values as bf16 = two 16-byte chunks (ch, ch+1) of row `row` of the
// 128B-swizzled tile at shared address `tile`.
__device__ __forceinline__ void st_row_bf16x16(uint32_t tile, uint32_t row, uint32_t ch,
                                               const float *v) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        uint4 w;
        w.x = pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]);
        w.y = pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]);
        w.z = pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]);
        w.w = pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]);
        sts128(tile + sw128_off(row, ch + q), w);
    }
}
// Multiply the 8 bf16 values of a 16-byte chunk by s.
__device__ __forceinline__ uint4 scale_bf16x8(uint4 w, float s) {
    uint32_t *wd = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float2 f = unpack_bf16x2(wd[q]);
        wd[q] = pack_bf16x2(f.x * s, f.y * s);
    }
    return w;
}

__device__ __forceinline__ void prefetch_l2(const void *ptr) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
}

// Multiply the 8 bf16 values of a 16-byte chunk by 8 factors (one per channel).
__device__ __forceinline__ uint4 scale_bf16x8v(uint4 w, const float4 f0, const float4 f1) {
    uint32_t *wd = reinterpret_cast<uint32_t *>(&w);
    const float f[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float2 v = unpack_bf16x2(wd[q]);
        wd[q] = pack_bf16x2(v.x * f[2 * q], v.y * f[2 * q + 1]);
    }
    return w;
}

// ---- warp-level tf32 products for the 16x16 blocks of the triangular inverse
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// acc (16x16 fp32, two m16n8 fragments) += A (16x16) * B (16x16); A, B fp32 in shared
// memory with row strides lda, ldb (elements).
__device__ __forceinline__ void mma16x16x16_tf32(float (&acc)[2][4], const float *A, int lda,
                                                 const float *B, int ldb, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
        const uint32_t a0 = to_tf32(A[g * lda + 8 * kk + t]);
        const uint32_t a1 = to_tf32(A[(g + 8) * lda + 8 * kk + t]);
        const uint32_t a2 = to_tf32(A[g * lda + 8 * kk + t + 4]);
        const uint32_t a3 = to_tf32(A[(g + 8) * lda + 8 * kk + t + 4]);
#pragma unroll
        for (int nh = 0; nh < 2; ++nh) {
            const uint32_t b0 = to_tf32(B[(8 * kk + t) * ldb + 8 * nh + g]);
            const uint32_t b1 = to_tf32(B[(8 * kk + t + 4) * ldb + 8 * nh + g]);
            asm volatile(
                "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
                "{%8,%9}, {%0,%1,%2,%3};"
                : "+f"(acc[nh][0]), "+f"(acc[nh][1]), "+f"(acc[nh][2]), "+f"(acc[nh][3])
                : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
        }
    }
}
// C (16x16, row stride ldc) = s * acc
__device__ __forceinline__ void store16_tile(const float (&acc)[2][4], float *C, int ldc, int lane,
                                             float s) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
        C[g * ldc + 8 * nh + 2 * t] = s * acc[nh][0];
        C[g * ldc + 8 * nh + 2 * t + 1] = s * acc[nh][1];
        C[(g + 8) * ldc + 8 * nh + 2 * t] = s * acc[nh][2];
        C[(g + 8) * ldc + 8 * nh + 2 * t + 1] = s * acc[nh][3];
    }
}

// 64x64 unit lower-triangular inverse T = (I + Lm)^-1 by 16x16 blocks, run by NT threads
// (e = 0 .. NT-1, NT a multiple of 32 and at least 128) that meet at named barrier BAR
// between the steps: 64 threads solve the diagonal blocks while the others clear the
// upper blocks, then up to three warps form the off-diagonal blocks.
template <uint32_t BAR, int NT>
__device__ void invert_unit_lower(const float *Lm, float *Tm, float *Zs, int e) {
    constexpr int S = kLmStride;
    if (e < 64) {
        const int b = e >> 4, c = e & 15;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == c) ? 1.f : 0.f;
#pragma unroll
        for (int r = 1; r < 16; ++r) {
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int j = 0; j < r; j += 2) {
                s0 = fmaf(Lm[(16 * b + r) * S + 16 * b + j], x[j], s0);
                if (j + 1 < r) s1 = fmaf(Lm[(16 * b + r) * S + 16 * b + j + 1], x[j + 1], s1);
            }
            if (r > c) x[r] = -(s0 + s1);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tm[(16 * b + r) * S + 16 * b + c] = x[r];
    } else {
        for (int idx = e - 64; idx < 6 * 256; idx += NT - 64) {
            const int blk = idx >> 8, r = (idx >> 4) & 15, cc = idx & 15;
            const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
            const int bj = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
            Tm[(16 * bi + r) * S + 16 * bj + cc] = 0.f;
        }
    }
    named_sync(BAR, NT);
    // Off-diagonal blocks, by distance d = i - j:  T_ij = -T_ii sum_{k=j}^{i-1} L_ik T_kj.
    // Each block is one warp's job on the legacy warp-level tensor-core path (tf32
    // m16n8k8, fp32 accumulate): the products are 16x16x16, too small for tcgen05.
    const int w = e >> 5, lane = e & 31;
    for (int d = 1; d < 4; ++d) {
        if (w < 4 - d) {
            const int bi = w + d, bj = w;
            float acc[2][4] = {};
            for (int k = bj; k < bi; ++k)
                mma16x16x16_tf32(acc, Lm + (16 * bi) * S + 16 * k, S, Tm + (16 * k) * S + 16 * bj, S,
                                 lane);
            float *Z = Zs + w * 272;
            store16_tile(acc, Z, 17, lane, 1.f);
            __syncwarp();
            float acc2[2][4] = {};
            mma16x16x16_tf32(acc2, Tm + (16 * bi) * S + 16 * bi, S, Z, 17, lane);
            store16_tile(acc2, Tm + (16 * bi) * S + 16 * bj, S, lane, -1.f);
        }
        named_sync(BAR, NT);
    }
}

// Row stride (floats) of the fp32 64x64 scratch matrices of invert_unit_lower_rec: 16-byte
// aligned rows (float4 access), and the warp-level tf32 fragment loads stay nearly free of
// bank conflicts.
constexpr uint32_t kTStride = 68;

// T = (I + Lm)^-1 for a strictly lower-triangular 64x64 Lm (fp32, row stride kTStride),
// by recursive 2x2 blocking: the four 16x16 diagonal blocks by substitution (one warp
// each, lane c solving column c), then inside each 32x32 half T_10 = -T_11 L_10 T_00 on
// 16x16 blocks, then for the whole matrix T_10 = -T_11 (L_10 T_00) on 32x32 blocks, four
// 16x16 tiles per product.  The block products run on the warp-level tensor cores (tf32
// m16n8k8, fp32 accumulate).  Only the lower triangle and the diagonal of Tm are written
// (the 16x16 diagonal blocks entirely); readers take the rest as zero.  Warps w = 0-3 of
// the NT threads (e = 0 .. NT-1) do the work; all NT meet at named barrier BAR between the
// levels.  Zs holds 4 x 272 floats.
template <uint32_t BAR, int NT>
__device__ void invert_unit_lower_rec(const float *Lm, float *Tm, float *Zs, int e) {
    constexpr int S = kTStride;
    const int w = e >> 5, lane = e & 31;
    if (w < 4 && lane < 16) {
        const int b = w, c = lane;
        const float *Lb = Lm + (16 * b) * S + 16 * b;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) x[r] = (r == c) ? 1.f : 0.f;
#pragma unroll
        for (int r = 1; r < 16; ++r) {
            float l[16];
#pragma unroll
            for (int q = 0; q < (r + 3) / 4; ++q) {
                const float4 f = *reinterpret_cast<const float4 *>(Lb + r * S + 4 * q);
                l[4 * q] = f.x;
                l[4 * q + 1] = f.y;
                l[4 * q + 2] = f.z;
                l[4 * q + 3] = f.w;
            }
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
            for (int j = 0; j < r; ++j) {
                if ((j & 3) == 0) a0 = fmaf(l[j], x[j], a0);
                if ((j & 3) == 1) a1 = fmaf(l[j], x[j], a1);
                if ((j & 3) == 2) a2 = fmaf(l[j], x[j], a2);
                if ((j & 3) == 3) a3 = fmaf(l[j], x[j], a3);
            }
            if (r > c) x[r] = -((a0 + a1) + (a2 + a3));
        }
        float *Tb = Tm + (16 * b) * S + 16 * b + c;
#pragma unroll
        for (int r = 0; r < 16; ++r) Tb[r * S] = x[r];
    }
    named_sync(BAR, NT);
    // inside each 32x32 half: T_{2p+1, 2p} = -T_{2p+1, 2p+1} (L_{2p+1, 2p} T_{2p, 2p})
    if (w < 2) {
        const int i = 2 * w + 1, j = 2 * w;
        float acc[2][4] = {};
        mma16x16x16_tf32(acc, Lm + (16 * i) * S + 16 * j, S, Tm + (16 * j) * S + 16 * j, S, lane);
        float *Z = Zs + w * 272;
        store16_tile(acc, Z, 17, lane, 1.f);
        __syncwarp();
        float acc2[2][4] = {};
        mma16x16x16_tf32(acc2, Tm + (16 * i) * S + 16 * i, S, Z, 17, lane);
        store16_tile(acc2, Tm + (16 * i) * S + 16 * j, S, lane, -1.f);
    }
    named_sync(BAR, NT);
    // Y = L_{10} T_{00} on 32x32 blocks: tile (i, j), i in {2, 3}, j in {0, 1}
    if (w < 4) {
        const int i = 2 + (w >> 1), j = w & 1;
        float acc[2][4] = {};
        for (int k = j; k < 2; ++k)
            mma16x16x16_tf32(acc, Lm + (16 * i) * S + 16 * k, S, Tm + (16 * k) * S + 16 * j, S, lane);
        store16_tile(acc, Zs + w * 272, 17, lane, 1.f);
    }
    named_sync(BAR, NT);
    // T_{10} = -T_{11} Y: tile (i, j) = -sum_{k=2}^{i} T_{ik} Y_{kj}
    if (w < 4) {
        const int i = 2 + (w >> 1), j = w & 1;
        float acc[2][4] = {};
        for (int k = 2; k <= i; ++k)
            mma16x16x16_tf32(acc, Tm + (16 * i) * S + 16 * k, S, Zs + ((k - 2) * 2 + j) * 272, 17, lane);
        store16_tile(acc, Tm + (16 * i) * S + 16 * j, S, lane, -1.f);
    }
    named_sync(BAR, NT);
}

}  // namespace tc
}  // namespace la

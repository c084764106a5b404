// backward.cu -- the prefill's backward pass for the scalar-gate modes (la_prefill_backward).
//
// Lesson page "Linear attention and hybrids": the chunked form of section "Three forms of
// one computation" is the one used for training on long texts, with the gated recurrence
// of section "Memory must forget: decay and gates",  S_t = a_t S_{t-1} + v_t k_t^T,
// o_t = S_t q_t.  Given cotangents dO and dS_T of the outputs and the final state, with the
// in-chunk log-gate prefix lam_t, g_t = exp(lam_t), D_tj = exp(lam_t - lam_j) (j <= t), the
// state S_c at the chunk's start and G = dL/dS at the chunk's end:
//
//   P   = (Q K^T) o D,   dP = (dO V^T) o D          (causal, C x C)
//   dQ  = diag(g) dO S_c + dP K
//   dK  = dP^T Q + diag(g_L / g) V G
//   dV  = P^T dO + diag(g_L / g) K G^T
//   dL/dS_c = g_L G + dO^T diag(g) Q               (carried to the previous chunk)
//   dlam_t = q_t . dq_t - k_t . dk_t  (+ <dS_T, S_T> at the last token);  the gate
//   gradient is d log a_t = sum_{u >= t} dlam_u, da_t = d log a_t / a_t.
//
// The last identity follows from differentiating the decay mask exp(lam_s - lam_j): lam_u
// enters with + where it is the reading position and with - where it is the written one.
//
// fp32 arithmetic on CUDA cores, 256 threads per CTA and one or two CTAs per (batch, head)
// (the d_k columns of S and G split between them): a forward sweep stores every chunk-start
// state in the caller's workspace, then a reverse sweep carries G back through the chunks;
// a small kernel finishes dV and the gate gradient.  Tiles live in shared memory with one
// float of row padding; the products are register-tiled (a thread holds up to 16 x 4
// outputs), so that each shared load feeds several FMAs.
#include "bwd_util.cuh"
#include "la_internal.cuh"

#include <cfloat>

namespace la {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kBwdC = 32;

// A head's d_k columns are split over SPLIT CTAs (2 at d_k = 128): each CTA owns DK/SPLIT
// columns of S and G, the products that stay within columns (dQ, dK, the state and G
// updates), and a share of those that sum over them (dV, dlam), which it adds into fp32
// accumulators in the workspace; a finishing kernel converts dV and takes the suffix sums.
template <int DK, int DV, int SPLIT>
struct BwdSmem {
    static constexpr int DKH = DK / SPLIT;
    static constexpr int kS = DV * (DKH + 1);
    static constexpr int kQ = kBwdC * (DK + 1);
    static constexpr int kV = kBwdC * (DV + 1);
    static constexpr int kP = kBwdC * (kBwdC + 1);
    static constexpr int kFloats = 2 * kS + 2 * kQ + 2 * kV + 2 * kP + 4 * kBwdC + 8;
    static constexpr size_t kBytes = sizeof(float) * kFloats;
};
template <int DK>
constexpr int bwd_split() { return DK == 128 ? 2 : 1; }

__device__ __forceinline__ float block_sum(float x, float *red) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = x;
    __syncthreads();
    float s = 0.f;
    for (int i = 0; i < kBwdThreads / 32; ++i) s += red[i];
    return s;
}

template <int DK, int DV, int SPLIT, typename IO>
__global__ void __launch_bounds__(kBwdThreads)
backward_kernel(int T, int gate_heads, const IO *__restrict__ q, const IO *__restrict__ k,
                const IO *__restrict__ v, const float *__restrict__ gate,
                const float *__restrict__ S0, const IO *__restrict__ dO,
                const float *__restrict__ dST, IO *__restrict__ dq, IO *__restrict__ dk,
                float *__restrict__ dS0, float *__restrict__ ws, float *__restrict__ dv_acc,
                float *__restrict__ dl_acc) {
    using L = BwdSmem<DK, DV, SPLIT>;
    constexpr int C = kBwdC, DKH = L::DKH, SK = DK + 1, SV = DV + 1, SH = DKH + 1, SP = C + 1;
    constexpr int NW = kBwdThreads / 32;       // 8 warps
    constexpr int RC = C / NW;                 // chunk rows per warp (4)
    constexpr int RS = DV / NW;                // state rows per warp (16 or 8)
    constexpr int NK = DKH / 32, NV = DV / 32; // columns per lane
    extern __shared__ float smem[];
    float *S = smem;             // [DV][DKH+1]  state (forward) / chunk-start state (reverse)
    float *G = S + L::kS;        // [DV][DKH+1]  dL/dS at the chunk's end
    float *Qs = G + L::kS;       // [C][DK+1]
    float *Ks = Qs + L::kQ;      // [C][DK+1]
    float *Vs = Ks + L::kQ;      // [C][DV+1]
    float *dOs = Vs + L::kV;     // [C][DV+1]
    float *P = dOs + L::kV;      // [C][C+1]
    float *dP = P + L::kP;       // [C][C+1]
    float *lam = dP + L::kP;     // [C]   in-chunk log-gate prefix
    float *gv = lam + C;         // [C]   g_t = exp(lam_t)
    float *dec = gv + C;         // [C]   g_L / g_t
    float *dl = dec + C;         // [C]   this CTA's share of dlam
    float *red = dl + C;         // [8]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t bh = blockIdx.x / SPLIT;
    const int kh = blockIdx.x % SPLIT, c0 = kh * DKH;   // this CTA's columns c0 .. c0 + DKH
    const int nch = (T + C - 1) / C;
    const size_t row0 = bh * (size_t)T;
    const float *gh = gate ? (gate_heads ? gate + bh % gate_heads : gate + row0) : nullptr;
    const int gt = gate_heads ? 0 : 1;
    float *wsh = ws + (size_t)blockIdx.x * (nch + 1) * DV * DKH;

    auto load_gates = [&](int t0, int Lc) {
        if (tid < C) lam[tid] = (gh && tid < Lc) ? logf(fmaxf(gh[(size_t)(t0 + tid) * gt], FLT_MIN)) : 0.f;
        __syncthreads();
        if (tid == 0)
            for (int i = 1; i < C; ++i) lam[i] += lam[i - 1];
        __syncthreads();
        if (tid < C) {
            gv[tid] = expf(lam[tid]);
            dec[tid] = expf(lam[Lc - 1] - lam[tid]);
        }
        __syncthreads();
    };
    auto load_rows = [&](const IO *src, float *dst, int t0, int Lc, int d, int stride) {
        for (int p = tid; p < C * d; p += kBwdThreads) {
            const int i = p / d, j = p % d;
            dst[i * stride + j] = i < Lc ? to_f32(src[(row0 + t0 + i) * d + j]) : 0.f;
        }
    };
    auto st_idx = [&](int p) { return (p / DKH) * SH + p % DKH; };       // p over DV x DKH
    auto gl_idx = [&](int p) { return (p / DKH) * DK + c0 + p % DKH; };  // into [DV][DK]

    // ---- forward sweep: chunk-start states (this CTA's columns) into the workspace
    for (int p = tid; p < DV * DKH; p += kBwdThreads) S[st_idx(p)] = S0 ? S0[bh * DV * DK + gl_idx(p)] : 0.f;
    __syncthreads();
    for (int c = 0; c <= nch; ++c) {
        for (int p = tid; p < DV * DKH; p += kBwdThreads) wsh[(size_t)c * DV * DKH + p] = S[st_idx(p)];
        if (c == nch) break;
        const int t0 = c * C, Lc = min(C, T - t0);
        load_rows(k, Ks, t0, Lc, DK, SK);
        load_rows(v, Vs, t0, Lc, DV, SV);
        load_gates(t0, Lc);   // (synchronises: every thread has stored S)
        // S <- g_L S + sum_j (dec_j v_j) k_j^T
        const float gL = gv[Lc - 1];
        float acc[RS][NK] = {};
        tile_mma<RS, NK, C>(acc, RS * warp, lane, [&](int i, int j) { return dec[j] * Vs[j * SV + i]; },
                            [&](int j, int cc) { return Ks[j * SK + c0 + cc]; });
#pragma unroll
        for (int i = 0; i < RS; ++i)
#pragma unroll
            for (int n = 0; n < NK; ++n) {
                float &x = S[(RS * warp + i) * SH + lane + 32 * n];
                x = fmaf(gL, x, acc[i][n]);
            }
        __syncthreads();
    }
    __syncthreads();

    // ---- reverse sweep
    // S holds this CTA's columns of S_T: its share of <dS_T, S_T> (dlam at the last token)
    float part = 0.f;
    for (int p = tid; p < DV * DKH; p += kBwdThreads) {
        const float g0 = dST ? dST[bh * DV * DK + gl_idx(p)] : 0.f;
        G[st_idx(p)] = g0;
        part = fmaf(g0, S[st_idx(p)], part);
    }
    const float final_dot = block_sum(part, red);
    if (tid == 0 && final_dot != 0.f) atomicAdd(&dl_acc[row0 + T - 1], final_dot);
    for (int c = nch - 1; c >= 0; --c) {
        const int t0 = c * C, Lc = min(C, T - t0);
        load_rows(q, Qs, t0, Lc, DK, SK);
        load_rows(k, Ks, t0, Lc, DK, SK);
        load_rows(v, Vs, t0, Lc, DV, SV);
        load_rows(dO, dOs, t0, Lc, DV, SV);
        for (int p = tid; p < DV * DKH; p += kBwdThreads) S[st_idx(p)] = wsh[(size_t)c * DV * DKH + p];
        if (tid < C) dl[tid] = 0.f;
        load_gates(t0, Lc);   // (synchronises)
        const float gL = gv[Lc - 1];
        // causal decayed score matrices P = (Q K^T) o D, dP = (dO V^T) o D (full rows)
        for (int p = tid; p < C * C; p += kBwdThreads) {
            const int t = p / C, j = p % C;
            float pv = 0.f, dpv = 0.f;
            if (t < Lc && j <= t) {
                const float dd = expf(lam[t] - lam[j]);
                float a1 = 0.f, a2 = 0.f;
                for (int cc = 0; cc < DK; ++cc) a1 = fmaf(Qs[t * SK + cc], Ks[j * SK + cc], a1);
                for (int i = 0; i < DV; ++i) a2 = fmaf(dOs[t * SV + i], Vs[j * SV + i], a2);
                pv = a1 * dd;
                dpv = a2 * dd;
            }
            P[t * SP + j] = pv;
            dP[t * SP + j] = dpv;
        }
        __syncthreads();
        const int r0 = RC * warp;   // this warp's chunk rows
        {   // dQ = diag(g) dO S_c + dP K   (this CTA's columns)
            float acc[RC][NK] = {};
            tile_mma<RC, NK, DV>(acc, r0, lane, [&](int t, int i) { return dOs[t * SV + i]; },
                                 [&](int i, int cc) { return S[i * SH + cc]; });
#pragma unroll
            for (int i = 0; i < RC; ++i)
#pragma unroll
                for (int n = 0; n < NK; ++n) acc[i][n] *= gv[r0 + i];
            tile_mma<RC, NK, C>(acc, r0, lane, [&](int t, int j) { return dP[t * SP + j]; },
                                [&](int j, int cc) { return Ks[j * SK + c0 + cc]; });
#pragma unroll
            for (int i = 0; i < RC; ++i) {
                const int t = r0 + i;
                float qd = 0.f;
#pragma unroll
                for (int n = 0; n < NK; ++n) {
                    const int cc = c0 + lane + 32 * n;
                    qd = fmaf(Qs[t * SK + cc], acc[i][n], qd);
                    if (t < Lc) dq[(row0 + t0 + t) * DK + cc] = from_f32<IO>(acc[i][n]);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) qd += __shfl_xor_sync(0xffffffffu, qd, off);
                if (lane == 0 && t < Lc) atomicAdd(&dl[t], qd);
            }
        }
        {   // dK = dP^T Q + diag(g_L / g) V G   (this CTA's columns)
            float acc[RC][NK] = {};
            tile_mma<RC, NK, DV>(acc, r0, lane, [&](int t, int i) { return Vs[t * SV + i]; },
                                 [&](int i, int cc) { return G[i * SH + cc]; });
#pragma unroll
            for (int i = 0; i < RC; ++i)
#pragma unroll
                for (int n = 0; n < NK; ++n) acc[i][n] *= dec[r0 + i];
            tile_mma<RC, NK, C>(acc, r0, lane, [&](int t, int s) { return dP[s * SP + t]; },
                                [&](int s, int cc) { return Qs[s * SK + c0 + cc]; });
#pragma unroll
            for (int i = 0; i < RC; ++i) {
                const int t = r0 + i;
                float kd = 0.f;
#pragma unroll
                for (int n = 0; n < NK; ++n) {
                    const int cc = c0 + lane + 32 * n;
                    kd = fmaf(Ks[t * SK + cc], acc[i][n], kd);
                    if (t < Lc) dk[(row0 + t0 + t) * DK + cc] = from_f32<IO>(acc[i][n]);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) kd += __shfl_xor_sync(0xffffffffu, kd, off);
                if (lane == 0 && t < Lc) atomicAdd(&dl[t], -kd);
            }
        }
        {   // dV = P^T dO + diag(g_L / g) K G^T: this CTA's columns' share, added up in fp32
            float acc[RC][NV] = {};
            tile_mma<RC, NV, DKH>(acc, r0, lane, [&](int t, int cc) { return Ks[t * SK + c0 + cc]; },
                                  [&](int cc, int i) { return G[i * SH + cc]; });
#pragma unroll
            for (int i = 0; i < RC; ++i)
#pragma unroll
                for (int n = 0; n < NV; ++n) acc[i][n] *= dec[r0 + i];
            if (kh == 0)
                tile_mma<RC, NV, C>(acc, r0, lane, [&](int t, int s) { return P[s * SP + t]; },
                                    [&](int s, int i) { return dOs[s * SV + i]; });
#pragma unroll
            for (int i = 0; i < RC; ++i) {
                const int t = r0 + i;
                if (t < Lc)
#pragma unroll
                    for (int n = 0; n < NV; ++n) {
                        float *dst = dv_acc + (row0 + t0 + t) * DV + lane + 32 * n;
                        if (SPLIT == 1) *dst = acc[i][n];
                        else atomicAdd(dst, acc[i][n]);
                    }
            }
        }
        __syncthreads();
        if (tid < Lc) {
            if (SPLIT == 1) dl_acc[row0 + t0 + tid] += dl[tid];
            else atomicAdd(&dl_acc[row0 + t0 + tid], dl[tid]);
        }
        // carry G to the chunk start: G <- g_L G + dO^T diag(g) Q   (this CTA's columns)
        {
            float acc[RS][NK] = {};
            tile_mma<RS, NK, C>(acc, RS * warp, lane, [&](int i, int t) { return gv[t] * dOs[t * SV + i]; },
                                [&](int t, int cc) { return Qs[t * SK + c0 + cc]; });
#pragma unroll
            for (int i = 0; i < RS; ++i)
#pragma unroll
                for (int n = 0; n < NK; ++n) {
                    float &x = G[(RS * warp + i) * SH + lane + 32 * n];
                    x = fmaf(gL, x, acc[i][n]);
                }
        }
        __syncthreads();
    }
    if (dS0)
        for (int p = tid; p < DV * DKH; p += kBwdThreads) dS0[bh * DV * DK + gl_idx(p)] = G[st_idx(p)];
}

// Per (batch, head): dV from its fp32 accumulator, and the gate gradient
// d log a_t = sum_{u >= t} dlam_u (a suffix scan over the sequence), da_t = d log a_t / a_t.
template <typename IO>
__global__ void __launch_bounds__(kBwdThreads)
backward_finish_kernel(int T, int DV, const float *__restrict__ dv_acc, IO *__restrict__ dv,
                       const float *__restrict__ dl_acc, const float *__restrict__ gate,
                       float *__restrict__ dgate) {
    __shared__ float tot[kBwdThreads];
    const size_t bh = blockIdx.x, row0 = bh * (size_t)T;
    const int tid = threadIdx.x;
    for (size_t e = tid; e < (size_t)T * DV; e += kBwdThreads)
        dv[row0 * DV + e] = from_f32<IO>(dv_acc[row0 * DV + e]);
    if (!dgate) return;
    const int per = (T + kBwdThreads - 1) / kBwdThreads;
    const int a0 = min(T, tid * per), a1 = min(T, a0 + per);
    float s = 0.f;
    for (int t = a0; t < a1; ++t) s += dl_acc[row0 + t];
    tot[tid] = s;
    __syncthreads();
    if (tid == 0) {   // exclusive suffix sums of the thread totals
        float run = 0.f;
        for (int i = kBwdThreads - 1; i >= 0; --i) {
            const float x = tot[i];
            tot[i] = run;
            run += x;
        }
    }
    __syncthreads();
    float run = tot[tid];
    for (int t = a1 - 1; t >= a0; --t) {
        run += dl_acc[row0 + t];
        dgate[row0 + t] = run / fmaxf(gate[row0 + t], FLT_MIN);
    }
}

template <int DK, int DV, typename IO>
cudaError_t launch_bwd(int BH, int T, int gate_heads, const void *q, const void *k, const void *v,
                       const float *gate, const float *S0, const void *dO, const float *dST,
                       void *dq, void *dk, void *dv, float *dgate, float *dS0, float *ws,
                       cudaStream_t st) {
    constexpr int SPLIT = bwd_split<DK>();
    using L = BwdSmem<DK, DV, SPLIT>;
    const size_t nch = ((size_t)T + kBwdC - 1) / kBwdC;
    float *dv_acc = ws + (size_t)BH * (nch + 1) * DV * DK;
    float *dl_acc = dv_acc + (size_t)BH * T * DV;
    cudaError_t e = cudaMemsetAsync(dv_acc, 0, sizeof(float) * (size_t)BH * T * (DV + 1), st);
    if (e != cudaSuccess) return e;
    auto kern = backward_kernel<DK, DV, SPLIT, IO>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kBytes);
    if (e != cudaSuccess) return e;
    timer_begin(st);
    kern<<<(unsigned)(BH * SPLIT), kBwdThreads, L::kBytes, st>>>(
        T, gate_heads, static_cast<const IO *>(q), static_cast<const IO *>(k), static_cast<const IO *>(v),
        gate, S0, static_cast<const IO *>(dO), dST, static_cast<IO *>(dq), static_cast<IO *>(dk), dS0,
        ws, dv_acc, dl_acc);
    timer_end(st);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    timer_begin(st);
    backward_finish_kernel<IO><<<(unsigned)BH, kBwdThreads, 0, st>>>(
        T, DV, dv_acc, static_cast<IO *>(dv), dl_acc, gate, dgate);
    timer_end(st);
    note_launches(2);
    return cudaGetLastError();
}

template <typename IO>
cudaError_t launch_dims_bwd(int dkd, int dvd, int BH, int T, int gh, const void *q, const void *k,
                            const void *v, const float *gate, const float *S0, const void *dO,
                            const float *dST, void *dq, void *dk, void *dv, float *dgate,
                            float *dS0, float *ws, cudaStream_t st) {
#define LA_BWD(A, B)                                                                          \
    if (dkd == A && dvd == B)                                                                 \
        return launch_bwd<A, B, IO>(BH, T, gh, q, k, v, gate, S0, dO, dST, dq, dk, dv, dgate, dS0, \
                                    ws, st);
    LA_BWD(64, 64)
    LA_BWD(128, 128)
    LA_BWD(64, 128)
    LA_BWD(128, 64)
#undef LA_BWD
    return cudaErrorInvalidValue;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// True if `p` is memory the current device can address.
bool on_device(const void *p) {
    if (!p) return false;
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        (void)cudaGetLastError();
        return false;
    }
    if (attr.type == cudaMemoryTypeManaged) return true;
    if (attr.type != cudaMemoryTypeDevice) return false;
    int dev = -1;
    return cudaGetDevice(&dev) == cudaSuccess && attr.device == dev;
}

}  // namespace
}  // namespace la

using namespace la;

extern "C" size_t la_backward_workspace_size(la_mode_t mode, int B, int H, int T, int d_k, int d_v) {
    if (mode == LA_MODE_GATED_DELTA || mode == LA_MODE_KDA)
        return delta_backward_workspace_bytes(mode, B, H, T, d_k, d_v);
    if ((mode != LA_MODE_GATED && mode != LA_MODE_RETNET) || B < 1 || H < 1 || T < 1) return 0;
    const size_t nch = ((size_t)T + kBwdC - 1) / kBwdC;
    // every chunk-start state, then the fp32 accumulators of dv and dlam
    return sizeof(float) * (size_t)B * H * ((nch + 1) * d_k * d_v + (size_t)T * (d_v + 1));
}

extern "C" la_status_t la_prefill_backward(la_mode_t mode, la_dtype_t dtype, int B, int H, int T,
                                           int d_k, int d_v, const void *q, const void *k,
                                           const void *v, const float *gate, const float *state0,
                                           const void *dO, const float *dstate, void *dq,
                                           void *dk, void *dv, float *dgate, float *dstate0,
                                           void *workspace, size_t workspace_bytes, void *stream) {
    timer_reset();
    if (mode < LA_MODE_ELU1_NORM || mode > LA_MODE_RETNET) return LA_ERR_INVALID_ARG;
    if (mode != LA_MODE_GATED && mode != LA_MODE_RETNET) return LA_ERR_UNSUPPORTED;
    if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || T < 1) return LA_ERR_INVALID_ARG;
    if (!((d_k == 64 || d_k == 128) && (d_v == 64 || d_v == 128))) return LA_ERR_UNSUPPORTED;
    const long long BH = (long long)B * H;
    if (BH > INT32_MAX || BH * T * (long long)(d_k > d_v ? d_k : d_v) > (1ll << 40)) return LA_ERR_INVALID_ARG;
    if (mode == LA_MODE_RETNET && (!gate || dgate)) return LA_ERR_INVALID_ARG;   // gamma is fixed
    if (mode == LA_MODE_GATED && dgate && !gate) return LA_ERR_INVALID_ARG;
    const void *need[] = {q, k, v, dO, dq, dk, dv};
    for (const void *p : need)
        if (!on_device(p) || !aligned16(p)) return LA_ERR_INVALID_ARG;
    const void *opt[] = {gate, state0, dstate, dgate, dstate0};
    for (const void *p : opt)
        if (p && (!on_device(p) || (reinterpret_cast<uintptr_t>(p) & 3u))) return LA_ERR_INVALID_ARG;
    const size_t need_ws = la_backward_workspace_size(mode, B, H, T, d_k, d_v);
    if (!workspace || workspace_bytes < need_ws || !on_device(workspace) || !aligned16(workspace))
        return LA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int gh = (mode == LA_MODE_RETNET) ? H : 0;
    float *ws = static_cast<float *>(workspace);
    const cudaError_t e =
        dtype == LA_BF16
            ? launch_dims_bwd<__nv_bfloat16>(d_k, d_v, (int)BH, T, gh, q, k, v, gate, state0, dO, dstate,
                                             dq, dk, dv, dgate, dstate0, ws, st)
            : launch_dims_bwd<float>(d_k, d_v, (int)BH, T, gh, q, k, v, gate, state0, dO, dstate, dq, dk,
                                     dv, dgate, dstate0, ws, st);
    return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

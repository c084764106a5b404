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
// One CTA (256 threads) per (batch, head), fp32 arithmetic on CUDA cores: a forward sweep
// stores every chunk-start state in the caller's workspace, then a reverse sweep carries G
// back through the chunks.  Tiles live in shared memory with one float of row padding.
#include "la_internal.cuh"

#include <cfloat>

namespace la {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kBwdC = 32;

template <int DK, int DV>
struct BwdSmem {
    static constexpr int kS = DV * (DK + 1);
    static constexpr int kQ = kBwdC * (DK + 1);
    static constexpr int kV = kBwdC * (DV + 1);
    static constexpr int kP = kBwdC * (kBwdC + 1);
    static constexpr int kFloats = 2 * kS + 2 * kQ + 2 * kV + 2 * kP + 4 * kBwdC + 8;
    static constexpr size_t kBytes = sizeof(float) * kFloats;
};

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

template <int DK, int DV, typename IO>
__global__ void __launch_bounds__(kBwdThreads)
backward_kernel(int T, int gate_heads, const IO *__restrict__ q, const IO *__restrict__ k,
                const IO *__restrict__ v, const float *__restrict__ gate,
                const float *__restrict__ S0, const IO *__restrict__ dO,
                const float *__restrict__ dST, IO *__restrict__ dq, IO *__restrict__ dk,
                IO *__restrict__ dv, float *__restrict__ dgate, float *__restrict__ dS0,
                float *__restrict__ ws) {
    using L = BwdSmem<DK, DV>;
    constexpr int C = kBwdC, SK = DK + 1, SV = DV + 1, SP = C + 1;
    extern __shared__ float smem[];
    float *S = smem;             // [DV][DK+1]  state (forward) / chunk-start state (reverse)
    float *G = S + L::kS;        // [DV][DK+1]  dL/dS at the chunk's end
    float *Qs = G + L::kS;       // [C][DK+1]
    float *Ks = Qs + L::kQ;      // [C][DK+1]
    float *Vs = Ks + L::kQ;      // [C][DV+1]
    float *dOs = Vs + L::kV;     // [C][DV+1]
    float *P = dOs + L::kV;      // [C][C+1]
    float *dP = P + L::kP;       // [C][C+1]
    float *lam = dP + L::kP;     // [C]
    float *dl = lam + C;         // [C]   dlam
    float *av = dl + C;          // [C]   gate values (clamped)
    float *dlr = av + C;         // [C]
    float *red = dlr + C;        // [8]

    const int tid = threadIdx.x;
    const size_t bh = blockIdx.x;
    const int nch = (T + C - 1) / C;
    const size_t row0 = bh * (size_t)T;
    const float *gh = gate ? (gate_heads ? gate + bh % gate_heads : gate + row0) : nullptr;
    const int gt = gate_heads ? 0 : 1;
    float *wsh = ws + bh * (size_t)(nch + 1) * DV * DK;

    auto load_gates = [&](int t0, int Lc) {
        if (tid < C) {
            const float a = (gh && tid < Lc) ? fmaxf(gh[(size_t)(t0 + tid) * gt], FLT_MIN) : 1.f;
            av[tid] = a;
            lam[tid] = logf(a);
        }
        __syncthreads();
        if (tid == 0)
            for (int i = 1; i < C; ++i) lam[i] += lam[i - 1];
        __syncthreads();
    };
    auto load_rows = [&](const IO *src, float *dst, int t0, int Lc, int d, int stride) {
        for (int p = tid; p < C * d; p += kBwdThreads) {
            const int i = p / d, j = p % d;
            dst[i * stride + j] = i < Lc ? to_f32(src[(row0 + t0 + i) * d + j]) : 0.f;
        }
    };

    // ---- forward sweep: chunk-start states into the workspace
    for (int p = tid; p < DV * DK; p += kBwdThreads) S[(p / DK) * SK + p % DK] = S0 ? S0[bh * DV * DK + p] : 0.f;
    __syncthreads();
    for (int c = 0; c <= nch; ++c) {
        for (int p = tid; p < DV * DK; p += kBwdThreads) wsh[(size_t)c * DV * DK + p] = S[(p / DK) * SK + p % DK];
        if (c == nch) break;
        const int t0 = c * C, Lc = min(C, T - t0);
        load_rows(k, Ks, t0, Lc, DK, SK);
        load_rows(v, Vs, t0, Lc, DV, SV);
        load_gates(t0, Lc);
        const float lL = lam[Lc - 1], gL = expf(lL);
        for (int p = tid; p < DV * DK; p += kBwdThreads) {
            const int i = p / DK, cc = p % DK;
            float acc = 0.f;
            for (int j = 0; j < Lc; ++j) acc = fmaf(expf(lL - lam[j]) * Vs[j * SV + i], Ks[j * SK + cc], acc);
            S[i * SK + cc] = fmaf(gL, S[i * SK + cc], acc);
        }
        __syncthreads();
    }
    __syncthreads();

    // ---- reverse sweep
    // S holds S_T: <dS_T, S_T> enters dlam at the last token
    float part = 0.f;
    for (int p = tid; p < DV * DK; p += kBwdThreads) {
        const float gv = dST ? dST[bh * DV * DK + p] : 0.f;
        G[(p / DK) * SK + p % DK] = gv;
        part = fmaf(gv, S[(p / DK) * SK + p % DK], part);
    }
    const float final_dot = block_sum(part, red);
    float R = 0.f;   // sum of dlam over the tokens after this chunk
    for (int c = nch - 1; c >= 0; --c) {
        const int t0 = c * C, Lc = min(C, T - t0);
        load_rows(q, Qs, t0, Lc, DK, SK);
        load_rows(k, Ks, t0, Lc, DK, SK);
        load_rows(v, Vs, t0, Lc, DV, SV);
        load_rows(dO, dOs, t0, Lc, DV, SV);
        for (int p = tid; p < DV * DK; p += kBwdThreads) S[(p / DK) * SK + p % DK] = wsh[(size_t)c * DV * DK + p];
        if (tid < C) dl[tid] = 0.f;
        load_gates(t0, Lc);   // (synchronises)
        const float lL = lam[Lc - 1], gL = expf(lL);
        // causal decayed score matrices
        for (int p = tid; p < C * C; p += kBwdThreads) {
            const int t = p / C, j = p % C;
            float pv = 0.f, dpv = 0.f;
            if (t < Lc && j <= t) {
                const float dec = expf(lam[t] - lam[j]);
                float a1 = 0.f, a2 = 0.f;
                for (int cc = 0; cc < DK; ++cc) a1 = fmaf(Qs[t * SK + cc], Ks[j * SK + cc], a1);
                for (int i = 0; i < DV; ++i) a2 = fmaf(dOs[t * SV + i], Vs[j * SV + i], a2);
                pv = a1 * dec;
                dpv = a2 * dec;
            }
            P[t * SP + j] = pv;
            dP[t * SP + j] = dpv;
        }
        __syncthreads();
        // dQ and dK (rows t, columns cc), with their share of dlam
        for (int p = tid; p < Lc * DK; p += kBwdThreads) {
            const int t = p / DK, cc = p % DK;
            float sd = 0.f, gv = 0.f;
            for (int i = 0; i < DV; ++i) {
                sd = fmaf(S[i * SK + cc], dOs[t * SV + i], sd);
                gv = fmaf(G[i * SK + cc], Vs[t * SV + i], gv);
            }
            float a = expf(lam[t]) * sd, b = expf(lL - lam[t]) * gv;
            for (int j = 0; j <= t; ++j) a = fmaf(dP[t * SP + j], Ks[j * SK + cc], a);
            for (int s = t; s < Lc; ++s) b = fmaf(dP[s * SP + t], Qs[s * SK + cc], b);
            dq[(row0 + t0 + t) * DK + cc] = from_f32<IO>(a);
            dk[(row0 + t0 + t) * DK + cc] = from_f32<IO>(b);
            atomicAdd(&dl[t], Qs[t * SK + cc] * a - Ks[t * SK + cc] * b);
        }
        // dV
        for (int p = tid; p < Lc * DV; p += kBwdThreads) {
            const int t = p / DV, i = p % DV;
            float gk = 0.f;
            for (int cc = 0; cc < DK; ++cc) gk = fmaf(G[i * SK + cc], Ks[t * SK + cc], gk);
            float b = expf(lL - lam[t]) * gk;
            for (int s = t; s < Lc; ++s) b = fmaf(P[s * SP + t], dOs[s * SV + i], b);
            dv[(row0 + t0 + t) * DV + i] = from_f32<IO>(b);
        }
        __syncthreads();
        // gate gradient: suffix sums of dlam
        if (tid == 0) {
            if (c == nch - 1) dl[Lc - 1] += final_dot;
            float run = R;
            for (int t = Lc - 1; t >= 0; --t) {
                run += dl[t];
                dlr[t] = run;
            }
            R = run;
        }
        __syncthreads();
        R = dlr[0];
        if (dgate && tid < Lc) dgate[row0 + t0 + tid] = dlr[tid] / av[tid];
        // carry G to the chunk start: G <- g_L G + dO^T diag(g) Q
        for (int p = tid; p < DV * DK; p += kBwdThreads) {
            const int i = p / DK, cc = p % DK;
            float acc = 0.f;
            for (int t = 0; t < Lc; ++t) acc = fmaf(expf(lam[t]) * dOs[t * SV + i], Qs[t * SK + cc], acc);
            G[i * SK + cc] = fmaf(gL, G[i * SK + cc], acc);
        }
        __syncthreads();
    }
    if (dS0)
        for (int p = tid; p < DV * DK; p += kBwdThreads) dS0[bh * DV * DK + p] = G[(p / DK) * SK + p % DK];
}

template <int DK, int DV, typename IO>
cudaError_t launch_bwd(int BH, int T, int gate_heads, const void *q, const void *k, const void *v,
                       const float *gate, const float *S0, const void *dO, const float *dST,
                       void *dq, void *dk, void *dv, float *dgate, float *dS0, float *ws,
                       cudaStream_t st) {
    using L = BwdSmem<DK, DV>;
    auto kern = backward_kernel<DK, DV, IO>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kBytes);
    if (e != cudaSuccess) return e;
    timer_begin(st);
    kern<<<(unsigned)BH, kBwdThreads, L::kBytes, st>>>(
        T, gate_heads, static_cast<const IO *>(q), static_cast<const IO *>(k), static_cast<const IO *>(v),
        gate, S0, static_cast<const IO *>(dO), dST, static_cast<IO *>(dq), static_cast<IO *>(dk),
        static_cast<IO *>(dv), dgate, dS0, ws);
    timer_end(st);
    note_launches(1);
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
    if ((mode != LA_MODE_GATED && mode != LA_MODE_RETNET) || B < 1 || H < 1 || T < 1) return 0;
    const size_t nch = ((size_t)T + kBwdC - 1) / kBwdC;
    return sizeof(float) * (size_t)B * H * (nch + 1) * d_k * d_v;
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

// backward_delta.cu -- the prefill's backward pass for the delta-rule modes
// (la_prefill_backward_delta): Gated DeltaNet (mode 2) and Kimi Delta Attention (mode 3).
//
// Lesson page "Delta rule and Gated DeltaNet": S_t = S_{t-1} A_t (I - b_t k_t k_t^T)
// + b_t v_t k_t^T with A_t = a_t I (Gated DeltaNet) or Diag(a_t) (Kimi Delta Attention),
// read as o_t = S_t q_t; lesson page "Linear attention and hybrids", section "Three forms of
// one computation": the chunked form is the one used for training.  Per chunk of C tokens,
// with the in-chunk prefix lam_t of log a (per channel in mode 3), g_t = exp(lam_t),
// Gam_tj = exp(lam_t - lam_j) for j <= t (per channel in mode 3), the state S at the chunk's
// start (d_v x d_k) and the chunk's WY form:
//
//   Kg = g o K,   Qg = g o Q,   Kl = (g_L / g) o K
//   A   = Gam-weighted Q K^T (j <= t),    Kgr = Gam-weighted K K^T (j < t)
//   T   = (I + diag(b) Kgr)^-1,   W = T diag(b) Kg,   U = T diag(b) V
//   E   = U - W S^T,   O = Qg S^T + A E,   S_next^T = diag(g_L) S^T + Kl^T E
//
// Reverse mode through these steps, with H = dL/dS_next^T (d_k x d_v):
//
//   dE  = A^T dO + Kl H,   dA = tril(dO E^T),   dW = -dE S,   dU = dE
//   dV  = diag(b) T^T dE,  dT = dW (diag(b) Kg)^T + dE (diag(b) V)^T  (strictly lower part)
//   dLm = -T^T dT T^T (strictly lower), for Lm = diag(b) Kgr
//   dL/dS^T = Qg^T dO + diag(g_L) H - W^T dE            (carried to the previous chunk)
//   dq  = g o (dO S) + [Gam dA] K
//   dk  = b g o (T^T dW) + [Gam diag(b) dLm] K                              (lam_t enters +)
//         + [Gam dA]^T Q + [Gam diag(b) dLm]^T K + (g_L / g) o (E H^T)     (lam_t enters -)
//   db_t = Kg_t . (T^T dW)_t + V_t . (T^T dE)_t + sum_j dLm_tj Kgr_tj
//
// [Gam M] X stands for sum_j M_tj Gam_tj x_j (per channel in mode 3).  Every gate enters
// through a factor exp(+lam) or exp(-lam), so dL/dlam = q o dq + k o (dk_plus - dk_minus),
// split as marked above, plus at the chunk's last token the terms of g_L:
// sum_t k_t o (g_L / g_t)(E H^T)_t + g_L o colsum(S o H^T).  lam is a prefix within the
// chunk (the state carries the rest), so d log a_t is the suffix sum of dL/dlam within the
// chunk, and da_t = d log a_t / a_t.
//
// fp32 arithmetic on CUDA cores.  The rows of S (the d_v axis) evolve independently, so a
// head's d_v is split into slices of 32 rows, one CTA each: a forward sweep stores every
// chunk-start state slice in the workspace, then a reverse sweep carries H back through the
// chunks.  Each CTA recomputes the chunk's d_v-independent factors (Kgr, T, W) and adds its
// slice's share of dq, dk, db and dL/dlam (sums over d_v) into fp32 accumulators; dv and the
// slice of dL/dS_0 are its own.  A finishing kernel converts dq and dk and takes the gate
// suffix sums.  Gated DeltaNet's Gam is one C x C table per chunk; Kimi's per-channel Gam is
// evaluated per product term (exp2 of the log-gate difference, no factor outside [0, 1]),
// exact for any gate and slower.
#include "bwd_util.cuh"
#include "la_internal.cuh"

#include <cfloat>

namespace la {
namespace {

constexpr int kDT = 256;            // threads per CTA (8 warps)
constexpr int kDC = 32;             // chunk length
constexpr int kDVS = 32;            // d_v rows per CTA
constexpr int kPC = kDC + 1;        // row pitch of C x C tiles
constexpr int kPV = kDVS + 1;       // row pitch of C x d_v-slice tiles

template <int MODE, int DK>
struct DeltaBwdSmem {
    static constexpr int PK = DK + 1;
    static constexpr int CK = kDC * PK;     // C x d_k tile
    static constexpr int SK = kDVS * PK;    // d_v slice x d_k tile
    static constexpr int CC = kDC * kPC;
    static constexpr int CV = kDC * kPV;
    // C x d_k: Qs Ks Wm dWm, and in mode 3 Lg (log2 gate prefix) Kg Kl Qg
    static constexpr int nCK = MODE == 3 ? 8 : 4;
    // C x C: Am Km Tm Xm (Lm, then dT T^T) dAm dTm Gm BL
    static constexpr int nCC = 8;
    // C x d_v slice: Vs dOs Es dEs TdE
    static constexpr int nCV = 5;
    // bet lam g dec dbl | gl col1 col2
    static constexpr int kSmall = 5 * kDC + 3 * DK;
    static constexpr int kFloats = nCK * CK + 2 * SK + nCC * CC + nCV * CV + kSmall;
    static constexpr size_t kBytes = sizeof(float) * kFloats;
    static_assert(kBytes <= 227 * 1024, "shared memory");
};

// Shared-memory views of one CTA's chunk.
template <int MODE, int DK>
struct ChunkTiles {
    using L = DeltaBwdSmem<MODE, DK>;
    static constexpr int PK = L::PK;
    float *Qs, *Ks, *Wm, *dWm, *Lg, *Kg, *Kl, *Qg;
    float *Ss, *Hs;
    float *Am, *Km, *Tm, *Xm, *dAm, *dTm, *Gm, *BL;
    float *Vs, *dOs, *Es, *dEs, *TdE;
    float *bet, *lam, *g, *dec, *dbl, *gl, *col1, *col2;

    __device__ explicit ChunkTiles(float *sm) {
        float *p = sm;
        auto take = [&](int n) { float *r = p; p += n; return r; };
        Qs = take(L::CK); Ks = take(L::CK); Wm = take(L::CK); dWm = take(L::CK);
        if constexpr (MODE == 3) {
            Lg = take(L::CK); Kg = take(L::CK); Kl = take(L::CK); Qg = take(L::CK);
        } else {
            Lg = Kg = Kl = Qg = nullptr;
        }
        Ss = take(L::SK); Hs = take(L::SK);
        Am = take(L::CC); Km = take(L::CC); Tm = take(L::CC); Xm = take(L::CC);
        dAm = take(L::CC); dTm = take(L::CC); Gm = take(L::CC); BL = take(L::CC);
        Vs = take(L::CV); dOs = take(L::CV); Es = take(L::CV); dEs = take(L::CV); TdE = take(L::CV);
        bet = take(kDC); lam = take(kDC); g = take(kDC); dec = take(kDC); dbl = take(kDC);
        gl = take(DK); col1 = take(DK); col2 = take(DK);
    }
    // Kg, Kl, Qg entries: per channel (mode 3) or the token's scalar factor (mode 2).
    __device__ __forceinline__ float kg(int t, int c) const {
        if constexpr (MODE == 3) return Kg[t * PK + c];
        else return Ks[t * PK + c] * g[t];
    }
    __device__ __forceinline__ float kl(int t, int c) const {
        if constexpr (MODE == 3) return Kl[t * PK + c];
        else return Ks[t * PK + c] * dec[t];
    }
    __device__ __forceinline__ float qg(int t, int c) const {
        if constexpr (MODE == 3) return Qg[t * PK + c];
        else return Qs[t * PK + c] * g[t];
    }
    __device__ __forceinline__ float gf(int t, int c) const {   // g_tc
        if constexpr (MODE == 3) return exp2f(Lg[t * PK + c]);
        else return g[t];
    }
    __device__ __forceinline__ float decf(int t, int c, int last) const {   // g_L / g_t
        if constexpr (MODE == 3) return exp2f(Lg[last * PK + c] - Lg[t * PK + c]);
        else return dec[t];
    }
};

// Rows [t0, t0 + n) of a [rows, d] tensor into a C x d tile (pitch `pitch`), columns
// [c0, c0 + w) of the source; rows n .. C-1 are zero.
template <typename IO>
__device__ __forceinline__ void load_tile(const IO *__restrict__ src, size_t row0, int ld, int c0, int w,
                                          int n, float *dst, int pitch) {
    for (int p = threadIdx.x; p < kDC * w; p += kDT) {
        const int t = p / w, j = p % w;
        dst[t * pitch + j] = t < n ? to_f32(src[(row0 + t) * ld + c0 + j]) : 0.f;
    }
}

// The chunk's gates: b (zero past the last token), the log2 gate prefix (held at its last
// value past the last token) and the derived factors.  Mode 2: lam, g, dec, gl[all] = g_L
// and the C x C table Gm = Gam; mode 3: Lg, gl, Kg, Kl (and Qg when `with_q`).
template <int MODE, int DK>
__device__ void load_gates(const ChunkTiles<MODE, DK> &c, const float *__restrict__ gate,
                           const float *__restrict__ beta, size_t row0, int n, bool with_q) {
    constexpr int PK = DK + 1;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (warp == 0) {
        c.bet[lane] = lane < n ? beta[row0 + lane] : 0.f;
        if constexpr (MODE != 3) {
            float x = (gate && lane < n) ? log2f(fmaxf(gate[row0 + lane], FLT_MIN)) : 0.f;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += y;
            }
            const float xl = __shfl_sync(0xffffffffu, x, n - 1);
            c.lam[lane] = x;
            c.g[lane] = exp2f(x);
            c.dec[lane] = exp2f(xl - x);
            const float gL = exp2f(xl);
            for (int i = lane; i < DK; i += 32) c.gl[i] = gL;
        }
    }
    if constexpr (MODE == 3) {
        if (tid < DK) {
            float acc = 0.f;
            for (int t = 0; t < kDC; ++t) {
                if (gate && t < n) acc += log2f(fmaxf(gate[(row0 + t) * DK + tid], FLT_MIN));
                c.Lg[t * PK + tid] = acc;
            }
            c.gl[tid] = exp2f(c.Lg[(n - 1) * PK + tid]);
        }
    }
    __syncthreads();
    if constexpr (MODE == 3) {
        for (int p = tid; p < kDC * DK; p += kDT) {
            const int t = p / DK, j = p % DK, i = t * PK + j;
            const float lg = c.Lg[i];
            const float e = exp2f(lg);
            c.Kg[i] = c.Ks[i] * e;
            c.Kl[i] = c.Ks[i] * exp2f(c.Lg[(n - 1) * PK + j] - lg);
            if (with_q) c.Qg[i] = c.Qs[i] * e;
        }
    } else {
        for (int p = tid; p < kDC * kDC; p += kDT) {
            const int t = p / kDC, j = p % kDC;
            c.Gm[t * kPC + j] = j <= t ? exp2f(c.lam[t] - c.lam[j]) : 0.f;
        }
    }
    __syncthreads();
}

// Gam-weighted Gram products of the chunk: A (Q K^T, j <= t; only when `with_a`) into Am
// and Kgr (K K^T, j < t) into Km, Lm = diag(b) Kgr into Xm.  Rows 4 w + i, column = lane.
template <int MODE, int DK>
__device__ void grams(const ChunkTiles<MODE, DK> &c, bool with_a) {
    constexpr int PK = DK + 1;
    const int lane = threadIdx.x & 31, r0 = 4 * (threadIdx.x >> 5);
    float aA[4][1] = {}, aK[4][1] = {};
    if constexpr (MODE == 3) {
        for (int cc = 0; cc < DK; ++cc) {
            const float kj = c.Ks[lane * PK + cc], lj = c.Lg[lane * PK + cc];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = r0 + i;
                const float e = lane <= t ? exp2f(c.Lg[t * PK + cc] - lj) : 0.f;
                const float ke = kj * e;
                if (with_a) aA[i][0] = fmaf(c.Qs[t * PK + cc], ke, aA[i][0]);
                aK[i][0] = fmaf(c.Ks[t * PK + cc], ke, aK[i][0]);
            }
        }
    } else {
        if (with_a)
            tile_mma<4, 1, DK>(aA, r0, lane, [&](int t, int cc) { return c.Qs[t * PK + cc]; },
                               [&](int cc, int j) { return c.Ks[j * PK + cc]; });
        tile_mma<4, 1, DK>(aK, r0, lane, [&](int t, int cc) { return c.Ks[t * PK + cc]; },
                           [&](int cc, int j) { return c.Ks[j * PK + cc]; });
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = r0 + i, j = lane;
        const float gm = MODE == 3 ? 1.f : c.Gm[t * kPC + j];
        if (with_a) c.Am[t * kPC + j] = j <= t ? aA[i][0] * gm : 0.f;
        const float kgr = j < t ? aK[i][0] * gm : 0.f;
        c.Km[t * kPC + j] = kgr;
        c.Xm[t * kPC + j] = c.bet[t] * kgr;
    }
}

// T = (I + Lm)^-1 for the strictly lower Lm in Xm, into Tm.  One warp: lane j holds column j
// in registers and the rows follow by forward substitution.
__device__ __forceinline__ void invert_unit_lower_32(const float *Lm, float *Tm) {
    const int lane = threadIdx.x & 31;
    float x[kDC];
#pragma unroll
    for (int i = 0; i < kDC; ++i) x[i] = i == lane ? 1.f : 0.f;
#pragma unroll
    for (int i = 1; i < kDC; ++i) {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int k = 0; k < i; ++k) {
            const float l = Lm[i * kPC + k];
            if (k & 1) s1 = fmaf(l, x[k], s1);
            else s0 = fmaf(l, x[k], s0);
        }
        if (i > lane) x[i] = -(s0 + s1);
    }
#pragma unroll
    for (int i = 0; i < kDC; ++i) Tm[i * kPC + lane] = x[i];
}

// W = T diag(b) Kg into Wm and U = T diag(b) V into Es (the chunk's WY factors).
template <int MODE, int DK>
__device__ __forceinline__ void wy_factors(const ChunkTiles<MODE, DK> &c) {
    constexpr int PK = DK + 1, NK = DK / 32;
    const int lane = threadIdx.x & 31, r0 = 4 * (threadIdx.x >> 5);
    auto tb = [&](int t, int u) { return c.Tm[t * kPC + u] * c.bet[u]; };
    float w[4][NK] = {};
    tile_mma<4, NK, kDC>(w, r0, lane, tb, [&](int u, int cc) { return c.kg(u, cc); });
    float uu[4][1] = {};
    tile_mma<4, 1, kDC>(uu, r0, lane, tb, [&](int u, int j) { return c.Vs[u * kPV + j]; });
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int n = 0; n < NK; ++n) c.Wm[(r0 + i) * PK + lane + 32 * n] = w[i][n];
        c.Es[(r0 + i) * kPV + lane] = uu[i][0];
    }
}

// E = U - W S^T, in place in Es (each thread updates the entries it wrote as U).
template <int MODE, int DK>
__device__ __forceinline__ void new_values(const ChunkTiles<MODE, DK> &c) {
    constexpr int PK = DK + 1;
    const int lane = threadIdx.x & 31, r0 = 4 * (threadIdx.x >> 5);
    float e[4][1] = {};
    tile_mma<4, 1, DK>(e, r0, lane, [&](int t, int cc) { return c.Wm[t * PK + cc]; },
                       [&](int cc, int j) { return c.Ss[j * PK + cc]; });
#pragma unroll
    for (int i = 0; i < 4; ++i) c.Es[(r0 + i) * kPV + lane] -= e[i][0];
}

// ---------------------------------------------------------------------------------------
// Forward sweep: every chunk-start state slice into the workspace.
template <int MODE, int DK, typename IO>
__global__ void __launch_bounds__(kDT)
delta_states_kernel(int T, int DV, const IO *__restrict__ k, const IO *__restrict__ v,
                    const float *__restrict__ gate, const float *__restrict__ beta,
                    const float *__restrict__ S0, float *__restrict__ states) {
    using L = DeltaBwdSmem<MODE, DK>;
    constexpr int PK = L::PK, NK = DK / 32;
    extern __shared__ float smem[];
    const ChunkTiles<MODE, DK> c(smem);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, r0 = 4 * warp;
    const int NS = DV / kDVS;
    const size_t bh = blockIdx.x / NS;
    const int j0 = (blockIdx.x % NS) * kDVS;
    const int nch = (T + kDC - 1) / kDC;
    const size_t row0 = bh * (size_t)T;

    for (int p = tid; p < kDVS * DK; p += kDT)
        c.Ss[(p / DK) * PK + p % DK] = S0 ? S0[(bh * DV + j0) * DK + p] : 0.f;
    __syncthreads();
    for (int ch = 0; ch < nch; ++ch) {
        const int t0 = ch * kDC, n = min(kDC, T - t0);
        float *dst = states + ((bh * nch + ch) * DV + j0) * (size_t)DK;
        for (int p = tid; p < kDVS * DK; p += kDT) dst[p] = c.Ss[(p / DK) * PK + p % DK];
        load_tile(k, row0 + t0, DK, 0, DK, n, c.Ks, PK);
        load_tile(v, row0 + t0, DV, j0, kDVS, n, c.Vs, kPV);
        __syncthreads();
        load_gates(c, gate, beta, row0 + t0, n, false);
        grams(c, false);
        __syncthreads();
        if (warp == 0) invert_unit_lower_32(c.Xm, c.Tm);
        __syncthreads();
        wy_factors(c);
        __syncthreads();
        new_values(c);
        __syncthreads();
        // S <- diag(g_L) S + E^T Kl  (rows j of this slice: warp-owned rows r0 + i)
        float s[4][NK] = {};
        tile_mma<4, NK, kDC>(s, r0, lane, [&](int j, int t) { return c.Es[t * kPV + j]; },
                             [&](int t, int cc) { return c.kl(t, cc); });
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int nn = 0; nn < NK; ++nn) {
                const int cc = lane + 32 * nn;
                float &x = c.Ss[(r0 + i) * PK + cc];
                x = fmaf(c.gl[cc], x, s[i][nn]);
            }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------------------
// Mode 3's Gam-weighted products, one term at a time (no factor outside [0, 1]).
// Row side: acc[i][n] += sum_{j <= t} M(t, j) X[j][c] 2^(Lg[t][c] - Lg[j][c]);
// column side: acc[i][n] += sum_{u >= t} M(u, t) X[u][c] 2^(Lg[u][c] - Lg[t][c]),
// for t = r0 + i and c = lane + 32 n.
template <int DK, typename FM>
__device__ __forceinline__ void gam_rows(float (&acc)[4][DK / 32], int r0, int lane, const float *Lg,
                                         const float *X, FM m) {
    constexpr int PK = DK + 1, NK = DK / 32;
    float lt[4][NK];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int n = 0; n < NK; ++n) lt[i][n] = Lg[(r0 + i) * PK + lane + 32 * n];
    for (int j = 0; j <= r0 + 3; ++j) {
#pragma unroll
        for (int n = 0; n < NK; ++n) {
            const float x = X[j * PK + lane + 32 * n], lj = Lg[j * PK + lane + 32 * n];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (j <= r0 + i) acc[i][n] = fmaf(m(r0 + i, j) * x, exp2f(lt[i][n] - lj), acc[i][n]);
        }
    }
}
template <int DK, typename FM>
__device__ __forceinline__ void gam_cols(float (&acc)[4][DK / 32], int r0, int lane, const float *Lg,
                                         const float *X, FM m) {
    constexpr int PK = DK + 1, NK = DK / 32;
    float lt[4][NK];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int n = 0; n < NK; ++n) lt[i][n] = Lg[(r0 + i) * PK + lane + 32 * n];
    for (int u = r0; u < kDC; ++u) {
#pragma unroll
        for (int n = 0; n < NK; ++n) {
            const float x = X[u * PK + lane + 32 * n], lu = Lg[u * PK + lane + 32 * n];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (u >= r0 + i) acc[i][n] = fmaf(m(u, r0 + i) * x, exp2f(lu - lt[i][n]), acc[i][n]);
        }
    }
}

// ---------------------------------------------------------------------------------------
// Reverse sweep.
template <int MODE, int DK, typename IO>
__global__ void __launch_bounds__(kDT)
delta_backward_kernel(int T, int DV, const IO *__restrict__ q, const IO *__restrict__ k,
                      const IO *__restrict__ v, const float *__restrict__ gate,
                      const float *__restrict__ beta, const IO *__restrict__ dO,
                      const float *__restrict__ dST, IO *__restrict__ dv, float *__restrict__ dS0,
                      const float *__restrict__ states, float *__restrict__ dq_acc,
                      float *__restrict__ dk_acc, float *__restrict__ dl_acc,
                      float *__restrict__ db_acc) {
    using L = DeltaBwdSmem<MODE, DK>;
    constexpr int PK = L::PK, NK = DK / 32;
    constexpr int DL = MODE == 3 ? DK : 1;   // entries of dL/dlam per token
    extern __shared__ float smem[];
    const ChunkTiles<MODE, DK> c(smem);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, r0 = 4 * warp;
    const int NS = DV / kDVS;
    const size_t bh = blockIdx.x / NS;
    const int j0 = (blockIdx.x % NS) * kDVS;
    const int nch = (T + kDC - 1) / kDC;
    const size_t row0 = bh * (size_t)T;

    for (int p = tid; p < kDVS * DK; p += kDT)
        c.Hs[(p / DK) * PK + p % DK] = dST ? dST[(bh * DV + j0) * DK + p] : 0.f;
    for (int ch = nch - 1; ch >= 0; --ch) {
        const int t0 = ch * kDC, n = min(kDC, T - t0), last = n - 1;
        const size_t r = row0 + t0;
        const float *src = states + ((bh * nch + ch) * DV + j0) * (size_t)DK;
        for (int p = tid; p < kDVS * DK; p += kDT) c.Ss[(p / DK) * PK + p % DK] = src[p];
        load_tile(q, r, DK, 0, DK, n, c.Qs, PK);
        load_tile(k, r, DK, 0, DK, n, c.Ks, PK);
        load_tile(v, r, DV, j0, kDVS, n, c.Vs, kPV);
        load_tile(dO, r, DV, j0, kDVS, n, c.dOs, kPV);
        if (tid < DK) c.col1[tid] = 0.f;
        __syncthreads();
        load_gates(c, gate, beta, r, n, true);
        grams(c, true);
        __syncthreads();

        // T (warp 0); the other warps meanwhile form dE = A^T dO + Kl H
        if (warp == 0) {
            invert_unit_lower_32(c.Xm, c.Tm);
        } else {
            for (int p = tid - 32; p < kDC * kDVS; p += kDT - 32) {
                const int t = p / kDVS, j = p % kDVS;
                float a0 = 0.f, a1 = 0.f;
                for (int u = t; u < kDC; ++u) a0 = fmaf(c.Am[u * kPC + t], c.dOs[u * kPV + j], a0);
                for (int cc = 0; cc < DK; ++cc) a1 = fmaf(c.kl(t, cc), c.Hs[j * PK + cc], a1);
                c.dEs[t * kPV + j] = a0 + a1;
            }
        }
        __syncthreads();
        wy_factors(c);
        __syncthreads();
        new_values(c);
        __syncthreads();

        {   // T^T dE (-> dv), dA = tril(dO E^T), dW = -dE S
            float td[4][1] = {}, da[4][1] = {}, dw[4][NK] = {};
            tile_mma<4, 1, kDC>(td, r0, lane, [&](int t, int u) { return c.Tm[u * kPC + t]; },
                                [&](int u, int j) { return c.dEs[u * kPV + j]; });
            tile_mma<4, 1, kDVS>(da, r0, lane, [&](int t, int i) { return c.dOs[t * kPV + i]; },
                                 [&](int i, int j) { return c.Es[j * kPV + i]; });
            tile_mma<4, NK, kDVS>(dw, r0, lane, [&](int t, int j) { return c.dEs[t * kPV + j]; },
                                  [&](int j, int cc) { return c.Ss[j * PK + cc]; });
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = r0 + i;
                c.TdE[t * kPV + lane] = td[i][0];
                if (t < n) dv[(r + t) * DV + j0 + lane] = from_f32<IO>(c.bet[t] * td[i][0]);
                c.dAm[t * kPC + lane] = lane <= t ? da[i][0] : 0.f;
#pragma unroll
                for (int nn = 0; nn < NK; ++nn) c.dWm[t * PK + lane + 32 * nn] = -dw[i][nn];
            }
        }
        __syncthreads();
        float tdw[4][NK] = {};
        {   // dT = (dW (diag(b)Kg)^T + dE (diag(b)V)^T), strictly lower; T^T dW (held)
            float dt[4][1] = {};
            tile_mma<4, 1, DK>(dt, r0, lane, [&](int t, int cc) { return c.dWm[t * PK + cc]; },
                               [&](int cc, int u) { return c.kg(u, cc); });
            tile_mma<4, 1, kDVS>(dt, r0, lane, [&](int t, int j) { return c.dEs[t * kPV + j]; },
                                 [&](int j, int u) { return c.Vs[u * kPV + j]; });
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = r0 + i;
                c.dTm[t * kPC + lane] = lane < t ? c.bet[lane] * dt[i][0] : 0.f;
            }
            tile_mma<4, NK, kDC>(tdw, r0, lane, [&](int t, int u) { return c.Tm[u * kPC + t]; },
                                 [&](int u, int cc) { return c.dWm[u * PK + cc]; });
        }
        __syncthreads();
        {   // X = dT T^T (over Lm, no longer needed); T^T dW over dW
            float x[4][1] = {};
            tile_mma<4, 1, kDC>(x, r0, lane, [&](int t, int u) { return c.dTm[t * kPC + u]; },
                                [&](int u, int j) { return c.Tm[j * kPC + u]; });
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                c.Xm[(r0 + i) * kPC + lane] = x[i][0];
#pragma unroll
                for (int nn = 0; nn < NK; ++nn) c.dWm[(r0 + i) * PK + lane + 32 * nn] = tdw[i][nn];
            }
        }
        __syncthreads();
        {   // dLm = -T^T X (strictly lower); BL = diag(b) dLm; mode 2 folds Gam into BL and dA
            float y[4][1] = {};
            tile_mma<4, 1, kDC>(y, r0, lane, [&](int t, int u) { return c.Tm[u * kPC + t]; },
                                [&](int u, int j) { return c.Xm[u * kPC + j]; });
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = r0 + i;
                const float dlm = lane < t ? -y[i][0] : 0.f;
                float part = dlm * c.Km[t * kPC + lane];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
                if (lane == 0) c.dbl[t] = part;
                const float gm = MODE == 3 ? 1.f : c.Gm[t * kPC + lane];
                c.BL[t * kPC + lane] = c.bet[t] * dlm * gm;
                if (MODE != 3) c.dAm[t * kPC + lane] *= gm;
            }
        }
        // (E H^T)-terms and the carried cotangent, both from H at the chunk's end
        float dkn[4][NK] = {}, hn[4][NK] = {};
        tile_mma<4, NK, kDVS>(dkn, r0, lane, [&](int t, int j) { return c.Es[t * kPV + j]; },
                              [&](int j, int cc) { return c.Hs[j * PK + cc]; });
#pragma unroll
        for (int nn = 0; nn < NK; ++nn) {
            const int cc = lane + 32 * nn;
            float s = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                dkn[i][nn] *= c.decf(r0 + i, cc, last);
                s = fmaf(c.Ks[(r0 + i) * PK + cc], dkn[i][nn], s);
            }
            atomicAdd(&c.col1[cc], s);
        }
        if (tid < DK) {
            float s = 0.f;
            for (int j = 0; j < kDVS; ++j) s = fmaf(c.Ss[j * PK + tid], c.Hs[j * PK + tid], s);
            c.col2[tid] = s;
        }
        {
            float h2[4][NK] = {};
            tile_mma<4, NK, kDC>(hn, r0, lane, [&](int j, int t) { return c.dOs[t * kPV + j]; },
                                 [&](int t, int cc) { return c.qg(t, cc); });
            tile_mma<4, NK, kDC>(h2, r0, lane, [&](int j, int t) { return c.dEs[t * kPV + j]; },
                                 [&](int t, int cc) { return c.Wm[t * PK + cc]; });
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int nn = 0; nn < NK; ++nn) {
                    const int cc = lane + 32 * nn;
                    hn[i][nn] = fmaf(c.gl[cc], c.Hs[(r0 + i) * PK + cc], hn[i][nn] - h2[i][nn]);
                }
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int nn = 0; nn < NK; ++nn) c.Hs[(r0 + i) * PK + lane + 32 * nn] = hn[i][nn];

        // dq, dk_plus, dk_minus
        float dq[4][NK] = {}, dkp[4][NK] = {};
        tile_mma<4, NK, kDVS>(dq, r0, lane, [&](int t, int j) { return c.dOs[t * kPV + j]; },
                              [&](int j, int cc) { return c.Ss[j * PK + cc]; });
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int nn = 0; nn < NK; ++nn) {
                const int t = r0 + i, cc = lane + 32 * nn;
                const float gtc = c.gf(t, cc);
                dq[i][nn] *= gtc;
                dkp[i][nn] = c.bet[t] * gtc * c.dWm[t * PK + cc];
            }
        if constexpr (MODE == 3) {
            gam_rows<DK>(dq, r0, lane, c.Lg, c.Ks, [&](int t, int j) { return c.dAm[t * kPC + j]; });
            gam_rows<DK>(dkp, r0, lane, c.Lg, c.Ks, [&](int t, int j) { return c.BL[t * kPC + j]; });
            gam_cols<DK>(dkn, r0, lane, c.Lg, c.Qs, [&](int u, int t) { return c.dAm[u * kPC + t]; });
            gam_cols<DK>(dkn, r0, lane, c.Lg, c.Ks, [&](int u, int t) { return c.BL[u * kPC + t]; });
        } else {
            tile_mma<4, NK, kDC>(dq, r0, lane, [&](int t, int j) { return c.dAm[t * kPC + j]; },
                                 [&](int j, int cc) { return c.Ks[j * PK + cc]; });
            tile_mma<4, NK, kDC>(dkp, r0, lane, [&](int t, int j) { return c.BL[t * kPC + j]; },
                                 [&](int j, int cc) { return c.Ks[j * PK + cc]; });
            tile_mma<4, NK, kDC>(dkn, r0, lane, [&](int t, int u) { return c.dAm[u * kPC + t]; },
                                 [&](int u, int cc) { return c.Qs[u * PK + cc]; });
            tile_mma<4, NK, kDC>(dkn, r0, lane, [&](int t, int u) { return c.BL[u * kPC + t]; },
                                 [&](int u, int cc) { return c.Ks[u * PK + cc]; });
        }
        __syncthreads();   // col1 complete

        // this slice's shares of dq, dk, dL/dlam and db, added into the fp32 accumulators
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = r0 + i;
            float dbs = 0.f, dls = 0.f;
#pragma unroll
            for (int nn = 0; nn < NK; ++nn) {
                const int cc = lane + 32 * nn;
                const float qv = c.Qs[t * PK + cc], kv = c.Ks[t * PK + cc];
                float dl = fmaf(qv, dq[i][nn], kv * (dkp[i][nn] - dkn[i][nn]));
                if (t == last) dl += c.col1[cc] + c.gl[cc] * c.col2[cc];
                dbs = fmaf(c.kg(t, cc), c.dWm[t * PK + cc], dbs);
                if (t < n) {
                    atomicAdd(&dq_acc[(r + t) * DK + cc], dq[i][nn]);
                    atomicAdd(&dk_acc[(r + t) * DK + cc], dkp[i][nn] + dkn[i][nn]);
                    if constexpr (DL > 1) atomicAdd(&dl_acc[(r + t) * DL + cc], dl);
                }
                dls += dl;
            }
            dbs = fmaf(c.Vs[t * kPV + lane], c.TdE[t * kPV + lane], dbs);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                dbs += __shfl_xor_sync(0xffffffffu, dbs, off);
                if constexpr (DL == 1) dls += __shfl_xor_sync(0xffffffffu, dls, off);
            }
            if (lane == 0 && t < n) {
                atomicAdd(&db_acc[r + t], dbs + c.dbl[t]);
                if constexpr (DL == 1) atomicAdd(&dl_acc[r + t], dls);
            }
        }
        __syncthreads();
    }
    if (dS0)
        for (int p = tid; p < kDVS * DK; p += kDT) dS0[(bh * DV + j0) * DK + p] = c.Hs[(p / DK) * PK + p % DK];
}

// dq, dk from their accumulators; db; the gate gradient from the suffix sums of dL/dlam
// within each chunk.  One CTA per (head row, chunk).
template <int MODE, int DK, typename IO>
__global__ void __launch_bounds__(128)
delta_finish_kernel(int T, const float *__restrict__ dq_acc, const float *__restrict__ dk_acc,
                    const float *__restrict__ dl_acc, const float *__restrict__ db_acc,
                    const float *__restrict__ gate, IO *__restrict__ dq, IO *__restrict__ dk,
                    float *__restrict__ dgate, float *__restrict__ dbeta) {
    const int nch = (T + kDC - 1) / kDC;
    const size_t bh = blockIdx.x / nch;
    const int ch = blockIdx.x % nch, t0 = ch * kDC, n = min(kDC, T - t0);
    const size_t r = bh * (size_t)T + t0;
    for (int p = threadIdx.x; p < n * DK; p += blockDim.x) {
        dq[r * DK + p] = from_f32<IO>(dq_acc[r * DK + p]);
        dk[r * DK + p] = from_f32<IO>(dk_acc[r * DK + p]);
    }
    if (dbeta && (int)threadIdx.x < n) dbeta[r + threadIdx.x] = db_acc[r + threadIdx.x];
    if (!dgate) return;
    constexpr int DL = MODE == 3 ? DK : 1;
    if ((int)threadIdx.x < DL) {
        float run = 0.f;
        for (int t = n - 1; t >= 0; --t) {
            const size_t e = (r + t) * DL + threadIdx.x;
            run += dl_acc[e];
            dgate[e] = run / fmaxf(gate[e], FLT_MIN);
        }
    }
}

struct DeltaWs {
    size_t states, dq, dk, dl, db, total;   // float offsets
};
DeltaWs delta_ws_layout(int mode, size_t BH, size_t T, size_t dk, size_t dv) {
    auto up = [](size_t x) { return (x + 3) & ~size_t(3); };
    const size_t nch = (T + kDC - 1) / kDC;
    DeltaWs w;
    w.states = 0;
    w.dq = up(BH * nch * dv * dk);
    w.dk = w.dq + up(BH * T * dk);
    w.dl = w.dk + up(BH * T * dk);
    w.db = w.dl + up(BH * T * (mode == LA_MODE_KDA ? dk : 1));
    w.total = w.db + up(BH * T);
    return w;
}

template <int MODE, int DK, typename IO>
cudaError_t launch_delta_bwd(int BH, int T, int DV, const void *q, const void *k, const void *v,
                             const float *gate, const float *beta, const float *S0, const void *dO,
                             const float *dST, void *dq, void *dk, void *dv, float *dgate,
                             float *dbeta, float *dS0, float *ws, cudaStream_t st) {
    using L = DeltaBwdSmem<MODE, DK>;
    const DeltaWs w = delta_ws_layout(MODE, BH, T, DK, DV);
    cudaError_t e = cudaMemsetAsync(ws + w.dq, 0, sizeof(float) * (w.total - w.dq), st);
    if (e != cudaSuccess) return e;
    auto fwd = delta_states_kernel<MODE, DK, IO>;
    auto rev = delta_backward_kernel<MODE, DK, IO>;
    e = cudaFuncSetAttribute(fwd, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kBytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(rev, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kBytes);
    if (e != cudaSuccess) return e;
    const unsigned ctas = (unsigned)(BH * (DV / kDVS));
    timer_begin(st);
    fwd<<<ctas, kDT, L::kBytes, st>>>(T, DV, static_cast<const IO *>(k), static_cast<const IO *>(v), gate,
                                      beta, S0, ws + w.states);
    timer_end(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    timer_begin(st);
    rev<<<ctas, kDT, L::kBytes, st>>>(T, DV, static_cast<const IO *>(q), static_cast<const IO *>(k),
                                      static_cast<const IO *>(v), gate, beta, static_cast<const IO *>(dO),
                                      dST, static_cast<IO *>(dv), dS0, ws + w.states, ws + w.dq, ws + w.dk,
                                      ws + w.dl, ws + w.db);
    timer_end(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const unsigned nch = (unsigned)((T + kDC - 1) / kDC);
    timer_begin(st);
    delta_finish_kernel<MODE, DK, IO><<<(unsigned)BH * nch, 128, 0, st>>>(
        T, ws + w.dq, ws + w.dk, ws + w.dl, ws + w.db, gate, static_cast<IO *>(dq), static_cast<IO *>(dk),
        dgate, dbeta);
    timer_end(st);
    note_launches(3);
    return cudaGetLastError();
}

template <typename IO>
cudaError_t launch_delta_dims(int mode, int dkd, int BH, int T, int DV, const void *q, const void *k,
                              const void *v, const float *gate, const float *beta, const float *S0,
                              const void *dO, const float *dST, void *dq, void *dk, void *dv,
                              float *dgate, float *dbeta, float *dS0, float *ws, cudaStream_t st) {
#define LA_DBWD(M, D)                                                                                \
    if (mode == M && dkd == D)                                                                       \
        return launch_delta_bwd<M, D, IO>(BH, T, DV, q, k, v, gate, beta, S0, dO, dST, dq, dk, dv, dgate, \
                                          dbeta, dS0, ws, st);
    LA_DBWD(2, 64)
    LA_DBWD(2, 128)
    LA_DBWD(3, 64)
    LA_DBWD(3, 128)
#undef LA_DBWD
    return cudaErrorInvalidValue;
}

bool dev_ok(const void *p, unsigned align) {
    if (!p || (reinterpret_cast<uintptr_t>(p) & (align - 1))) return false;
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

size_t delta_backward_workspace_bytes(int mode, int B, int H, int T, int d_k, int d_v) {
    if ((mode != LA_MODE_GATED_DELTA && mode != LA_MODE_KDA) || B < 1 || H < 1 || T < 1) return 0;
    return sizeof(float) * delta_ws_layout(mode, (size_t)B * H, T, d_k, d_v).total;
}

}  // namespace la

using namespace la;

extern "C" la_status_t la_prefill_backward_delta(la_mode_t mode, la_dtype_t dtype, int B, int H, int T,
                                                 int d_k, int d_v, const void *q, const void *k,
                                                 const void *v, const float *gate, const float *beta,
                                                 const float *state0, const void *dO, const float *dstate,
                                                 void *dq, void *dk, void *dv, float *dgate, float *dbeta,
                                                 float *dstate0, void *workspace, size_t workspace_bytes,
                                                 void *stream) {
    timer_reset();
    if (mode < LA_MODE_ELU1_NORM || mode > LA_MODE_RETNET) return LA_ERR_INVALID_ARG;
    if (mode != LA_MODE_GATED_DELTA && mode != LA_MODE_KDA) return LA_ERR_UNSUPPORTED;
    if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || T < 1) return LA_ERR_INVALID_ARG;
    if (!((d_k == 64 || d_k == 128) && (d_v == 64 || d_v == 128))) return LA_ERR_UNSUPPORTED;
    const long long BH = (long long)B * H;
    if (BH > INT32_MAX || BH * T * (long long)(d_k > d_v ? d_k : d_v) > (1ll << 40)) return LA_ERR_INVALID_ARG;
    if (dgate && !gate) return LA_ERR_INVALID_ARG;
    const void *need16[] = {q, k, v, dO, dq, dk, dv, workspace};
    for (const void *p : need16)
        if (!dev_ok(p, 16)) return LA_ERR_INVALID_ARG;
    if (!dev_ok(beta, 4)) return LA_ERR_INVALID_ARG;
    const void *opt[] = {gate, state0, dstate, dgate, dbeta, dstate0};
    for (const void *p : opt)
        if (p && !dev_ok(p, 4)) return LA_ERR_INVALID_ARG;
    const size_t need_ws = delta_backward_workspace_bytes(mode, B, H, T, d_k, d_v);
    if (workspace_bytes < need_ws) return LA_ERR_INVALID_ARG;
    const size_t es = dtype == LA_BF16 ? 2 : 4, th = (size_t)BH * T;
    const size_t gb = sizeof(float) * th * (mode == LA_MODE_KDA ? d_k : 1), sb = sizeof(float) * BH * d_v * d_k;
    if (!writes_disjoint({{dq, th * d_k * es}, {dk, th * d_k * es}, {dv, th * d_v * es}, {dgate, gb},
                          {dbeta, sizeof(float) * th}, {dstate0, sb}, {workspace, need_ws}},
                         {{q, th * d_k * es}, {k, th * d_k * es}, {v, th * d_v * es}, {dO, th * d_v * es},
                          {gate, gb}, {beta, sizeof(float) * th}, {state0, sb}, {dstate, sb}}))
        return LA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float *ws = static_cast<float *>(workspace);
    const cudaError_t e =
        dtype == LA_BF16
            ? launch_delta_dims<__nv_bfloat16>(mode, d_k, (int)BH, T, d_v, q, k, v, gate, beta, state0, dO,
                                               dstate, dq, dk, dv, dgate, dbeta, dstate0, ws, st)
            : launch_delta_dims<float>(mode, d_k, (int)BH, T, d_v, q, k, v, gate, beta, state0, dO, dstate,
                                       dq, dk, dv, dgate, dbeta, dstate0, ws, st);
    return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

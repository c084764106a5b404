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
// The rows of S (the d_v axis) evolve independently, so a head's d_v is split into slices
// of 32 rows, one CTA each: a forward sweep stores every chunk-start state slice in the
// workspace, then a reverse sweep carries H back through the chunks.  Each CTA recomputes
// the chunk's d_v-independent factors (Kgr, T, W) and adds its slice's share of dq, dk, db
// and dL/dlam (sums over d_v) into fp32 accumulators; dv and the slice of dL/dS_0 are its
// own.  A finishing kernel converts dq and dk and takes the gate suffix sums.
//
// The products run on the tensor cores as warp-level mma (m16n8k8, tf32 operands, fp32
// accumulate): the tiles are 32 x 32 and 32 x d_k, too small and too many for tcgen05's
// 128-row tiles, and each is followed by an element-wise step.  For fp32 I/O each operand
// is split into a tf32 part and a tf32 remainder (three products, fp32 accuracy); for
// bf16 I/O one tf32 product.  Gated DeltaNet's Gam is one C x C table per chunk folded into
// the coefficient matrices; Kimi's per-channel Gam is evaluated per term on the CUDA cores
// (exp2 of the log-gate difference, no factor outside [0, 1]), exact for any gate.
#include "la_internal.cuh"
#include "bwd_util.cuh"

#include <cfloat>
#include <type_traits>

namespace la {
namespace {

constexpr int kDT = 256;            // threads per CTA (8 warps)
constexpr int kDC = 32;             // chunk length
constexpr int kDVS = 32;            // d_v rows per CTA
// Row pitches are 4 (mod 32) floats: the mma operand loads of a row-major tile
// (row g, column t4 of a fragment) then fall in 32 distinct banks.
constexpr int kPC = kDC + 4;        // C x C tiles
constexpr int kPV = kDVS + 4;       // C x d_v-slice tiles
template <int DK> __host__ __device__ constexpr int pitch_k() { return DK + 4; }

template <int MODE, int DK>
struct DeltaBwdSmem {
    static constexpr int PK = pitch_k<DK>();
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
    // bet lam g dec dbl dbs dls | gl col1 col2
    static constexpr int kSmall = 7 * kDC + 3 * DK;
    // Gated DeltaNet stages the next chunk's raw inputs with cp.async while the current one
    // is processed (Kimi's per-channel tiles leave no room): q, k [C][d_k], v, dO [C][32]
    // in the I/O dtype (sized for 4-byte elements), the state slice [32][d_k], gate and b.
    static constexpr bool kStage = MODE != 3;
    static constexpr int kStageFloats = kStage ? 2 * kDC * DK + 2 * kDC * kDVS + kDVS * DK + 2 * kDC : 0;
    static constexpr int kFloats = nCK * CK + 2 * SK + nCC * CC + nCV * CV + kSmall + kStageFloats;
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
    float *bet, *lam, *g, *dec, *dbl, *dbs, *dls, *gl, *col1, *col2;
    float *sq, *sk, *sv, *sdo, *sS, *sg, *sb;   // staging (raw I/O elements in sq .. sdo)

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
        dbs = take(kDC); dls = take(kDC);
        gl = take(DK); col1 = take(DK); col2 = take(DK);
        if constexpr (L::kStage) {
            sq = take(kDC * DK); sk = take(kDC * DK); sv = take(kDC * kDVS); sdo = take(kDC * kDVS);
            sS = take(kDVS * DK); sg = take(kDC); sb = take(kDC);
        } else {
            sq = sk = sv = sdo = sS = sg = sb = nullptr;
        }
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

// Fragment ownership of the warp products (bwd_util.cuh's warp_mma): a 32 x 32 output
// gives warp w rows 16 (w & 1) .. +15 and columns 8 (w >> 1) .. +7 (one n-tile); a
// 32 x d_k output gives it rows 16 (w & 1) .. +15 and d_k / 4 columns from
// (d_k / 4)(w >> 1) (d_k / 32 n-tiles).  frag_each visits a thread's elements.
struct Own {
    int m0, n32, nk;
};
template <int DK>
__device__ __forceinline__ Own ownership() {
    const int w = threadIdx.x >> 5;
    return {16 * (w & 1), 8 * (w >> 1), (DK / 4) * (w >> 1)};
}
template <int NT, typename F>
__device__ __forceinline__ void frag_each(float (&d)[NT][4], int m0, int n0, F f) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) f(d[nt][r], m0 + g + 8 * (r >> 1), n0 + 8 * nt + 2 * t4 + (r & 1));
}

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

// One chunk's raw inputs into the staging buffers: k, v (columns j0 ..), gate, b, and for
// the reverse sweep q, dO and the chunk-start state slice; rows [0, n).
template <int MODE, int DK, typename IO>
__device__ __forceinline__ void stage_chunk(const ChunkTiles<MODE, DK> &c, const IO *q, const IO *k,
                                            const IO *v, const IO *dO, const float *gate,
                                            const float *beta, const float *state, size_t r, int n,
                                            int DV, int j0) {
    stage_rows<kDT>(c.sk, k + r * DK, DK, DK, n);
    stage_rows<kDT>(c.sv, v + r * DV + j0, DV, kDVS, n);
    if (q) {
        stage_rows<kDT>(c.sq, q + r * DK, DK, DK, n);
        stage_rows<kDT>(c.sdo, dO + r * DV + j0, DV, kDVS, n);
        stage_rows<kDT>(c.sS, state, DK, DK, kDVS);
    }
    const int tid = threadIdx.x;
    if (tid < n) cp_async4(c.sb + tid, beta + r + tid);
    if (gate && tid >= 32 && tid - 32 < n) cp_async4(c.sg + tid - 32, gate + r + tid - 32);
    cp_async_commit();
}
// The chunk's gates: b (zero past the last token), the log2 gate prefix (held at its last
// value past the last token) and the derived factors.  Mode 2: lam, g, dec, gl[all] = g_L
// and the C x C table Gm = Gam; mode 3: Lg, gl, Kg, Kl (and Qg when `with_q`).
// gate and beta point at the chunk's first token (global memory or the staging buffers).
template <int MODE, int DK>
__device__ void load_gates(const ChunkTiles<MODE, DK> &c, const float *gate, const float *beta, int n,
                           bool with_q) {
    constexpr int PK = pitch_k<DK>();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (warp == 0) {
        c.bet[lane] = lane < n ? beta[lane] : 0.f;
        if constexpr (MODE != 3) {
            float x = (gate && lane < n) ? log2f(fmaxf(gate[lane], FLT_MIN)) : 0.f;
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
                if (gate && t < n) acc += log2f(fmaxf(gate[t * DK + tid], FLT_MIN));
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
// and Kgr (K K^T, j < t) into Km, Lm = diag(b) Kgr into Xm.  Mode 2: tensor-core products
// scaled by the Gam table; mode 3: one exponential per term on the CUDA cores (rows
// 4 w + i, column = lane).
template <int MODE, int DK, bool SP>
__device__ void grams(const ChunkTiles<MODE, DK> &c, bool with_a) {
    constexpr int PK = pitch_k<DK>();
    const int lane = threadIdx.x & 31;
    if constexpr (MODE == 3) {
        const int r0 = 4 * (threadIdx.x >> 5);
        float aA[4] = {}, aK[4] = {};
        for (int cc = 0; cc < DK; ++cc) {
            const float kj = c.Ks[lane * PK + cc], lj = c.Lg[lane * PK + cc];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = r0 + i;
                const float e = lane <= t ? exp2f(c.Lg[t * PK + cc] - lj) : 0.f;
                const float ke = kj * e;
                if (with_a) aA[i] = fmaf(c.Qs[t * PK + cc], ke, aA[i]);
                aK[i] = fmaf(c.Ks[t * PK + cc], ke, aK[i]);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = r0 + i, j = lane;
            if (with_a) c.Am[t * kPC + j] = j <= t ? aA[i] : 0.f;
            const float kgr = j < t ? aK[i] : 0.f;
            c.Km[t * kPC + j] = kgr;
            c.Xm[t * kPC + j] = c.bet[t] * kgr;
        }
    } else {
        const Own o = ownership<DK>();
        float ak[1][4] = {};
        warp_mma<1, DK, SP>(ak, o.m0, o.n32, [&](int t, int cc) { return c.Ks[t * PK + cc]; },
                            [&](int cc, int j) { return c.Ks[j * PK + cc]; });
        frag_each(ak, o.m0, o.n32, [&](float &v, int t, int j) {
            const float kgr = j < t ? v * c.Gm[t * kPC + j] : 0.f;
            c.Km[t * kPC + j] = kgr;
            c.Xm[t * kPC + j] = c.bet[t] * kgr;
        });
        if (with_a) {
            float aa[1][4] = {};
            warp_mma<1, DK, SP>(aa, o.m0, o.n32, [&](int t, int cc) { return c.Qs[t * PK + cc]; },
                                [&](int cc, int j) { return c.Ks[j * PK + cc]; });
            frag_each(aa, o.m0, o.n32,
                      [&](float &v, int t, int j) { c.Am[t * kPC + j] = v * c.Gm[t * kPC + j]; });
        }
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

// W = T diag(b) Kg into Wm, U = T diag(b) V into Es and, with `with_de`,
// dE = A^T dO + Kl H into dEs.
template <int MODE, int DK, bool SP>
__device__ __forceinline__ void wy_factors(const ChunkTiles<MODE, DK> &c, bool with_de) {
    constexpr int PK = pitch_k<DK>(), NK = DK / 32;
    const Own o = ownership<DK>();
    auto tb = [&](int t, int u) { return c.Tm[t * kPC + u] * c.bet[u]; };
    float w[NK][4] = {};
    warp_mma<NK, kDC, SP>(w, o.m0, o.nk, tb, [&](int u, int cc) { return c.kg(u, cc); });
    frag_each(w, o.m0, o.nk, [&](float &v, int t, int cc) { c.Wm[t * PK + cc] = v; });
    float uu[1][4] = {};
    warp_mma<1, kDC, SP>(uu, o.m0, o.n32, tb, [&](int u, int j) { return c.Vs[u * kPV + j]; });
    frag_each(uu, o.m0, o.n32, [&](float &v, int t, int j) { c.Es[t * kPV + j] = v; });
    if (with_de) {
        float de[1][4] = {};
        warp_mma<1, kDC, SP>(de, o.m0, o.n32, [&](int t, int u) { return c.Am[u * kPC + t]; },
                             [&](int u, int j) { return c.dOs[u * kPV + j]; });
        warp_mma<1, DK, SP>(de, o.m0, o.n32, [&](int t, int cc) { return c.kl(t, cc); },
                            [&](int cc, int j) { return c.Hs[j * PK + cc]; });
        frag_each(de, o.m0, o.n32, [&](float &v, int t, int j) { c.dEs[t * kPV + j] = v; });
    }
}

// E = U - W S^T, in place in Es (each thread updates the entries it wrote as U).
template <int MODE, int DK, bool SP>
__device__ __forceinline__ void new_values(const ChunkTiles<MODE, DK> &c) {
    constexpr int PK = pitch_k<DK>();
    const Own o = ownership<DK>();
    float e[1][4] = {};
    warp_mma<1, DK, SP>(e, o.m0, o.n32, [&](int t, int cc) { return c.Wm[t * PK + cc]; },
                        [&](int cc, int j) { return c.Ss[j * PK + cc]; });
    frag_each(e, o.m0, o.n32, [&](float &v, int t, int j) { c.Es[t * kPV + j] -= v; });
}

// ---------------------------------------------------------------------------------------
// Forward sweep: every chunk-start state slice into the workspace.
template <int MODE, int DK, typename IO>
__global__ void __launch_bounds__(kDT)
delta_states_kernel(int T, int DV, const IO *__restrict__ k, const IO *__restrict__ v,
                    const float *__restrict__ gate, const float *__restrict__ beta,
                    const float *__restrict__ S0, float *__restrict__ states) {
    using L = DeltaBwdSmem<MODE, DK>;
    constexpr bool SP = std::is_same<IO, float>::value;
    constexpr int PK = L::PK, NK = DK / 32;
    extern __shared__ float smem[];
    const ChunkTiles<MODE, DK> c(smem);
    const int tid = threadIdx.x, warp = tid >> 5;
    const Own o = ownership<DK>();
    const int NS = DV / kDVS;
    const size_t bh = blockIdx.x / NS;
    const int j0 = (blockIdx.x % NS) * kDVS;
    const int nch = (T + kDC - 1) / kDC;
    const size_t row0 = bh * (size_t)T;

    for (int p = tid; p < kDVS * DK; p += kDT)
        c.Ss[(p / DK) * PK + p % DK] = S0 ? S0[(bh * DV + j0) * DK + p] : 0.f;
    __syncthreads();
    constexpr bool kStage = L::kStage;
    constexpr int GW = MODE == 3 ? DK : 1;   // gate floats per token
    auto stage = [&](int chs) {
        const int ts = chs * kDC;
        stage_chunk(c, static_cast<const IO *>(nullptr), k, v, static_cast<const IO *>(nullptr), gate, beta,
                    nullptr, row0 + ts, min(kDC, T - ts), DV, j0);
    };
    if constexpr (kStage) stage(0);
    for (int ch = 0; ch < nch; ++ch) {
        const int t0 = ch * kDC, n = min(kDC, T - t0);
        float *dst = states + ((bh * nch + ch) * DV + j0) * (size_t)DK;
        for (int p = tid; p < kDVS * DK; p += kDT) dst[p] = c.Ss[(p / DK) * PK + p % DK];
        if constexpr (kStage) {
            cp_async_wait_all();
            __syncthreads();
            unstage<kDT, IO>(c.sk, kDC, DK, n, c.Ks, PK);
            unstage<kDT, IO>(c.sv, kDC, kDVS, n, c.Vs, kPV);
        } else {
            load_tile(k, row0 + t0, DK, 0, DK, n, c.Ks, PK);
            load_tile(v, row0 + t0, DV, j0, kDVS, n, c.Vs, kPV);
        }
        __syncthreads();
        if constexpr (kStage) {
            load_gates(c, gate ? c.sg : nullptr, c.sb, n, false);
            if (ch + 1 < nch) stage(ch + 1);   // the staging buffers have been read
        } else {
            load_gates(c, gate ? gate + (row0 + t0) * GW : nullptr, beta + row0 + t0, n, false);
        }
        grams<MODE, DK, SP>(c, false);
        __syncthreads();
        if (warp == 0) invert_unit_lower_32(c.Xm, c.Tm);
        __syncthreads();
        wy_factors<MODE, DK, SP>(c, false);
        __syncthreads();
        new_values<MODE, DK, SP>(c);
        __syncthreads();
        // S <- diag(g_L) S + E^T Kl  (this slice's rows j; Ss is not read in this step)
        float s[NK][4] = {};
        warp_mma<NK, kDC, SP>(s, o.m0, o.nk, [&](int j, int t) { return c.Es[t * kPV + j]; },
                              [&](int t, int cc) { return c.kl(t, cc); });
        frag_each(s, o.m0, o.nk, [&](float &val, int j, int cc) {
            float &x = c.Ss[j * PK + cc];
            x = fmaf(c.gl[cc], x, val);
        });
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------------------
// Mode 3's Gam-weighted products, one term at a time (no factor outside [0, 1]), over a
// thread's fragment elements (t, c):
// row side     acc += sum_{j <= t} M(t, j) X[j][c] 2^(Lg[t][c] - Lg[j][c]),
// column side  acc += sum_{u >= t} M(u, t) X[u][c] 2^(Lg[u][c] - Lg[t][c]).
template <int NT, int DK, typename FM>
__device__ __forceinline__ void gam_rows(float (&acc)[NT][4], int m0, int n0, const float *Lg,
                                         const float *X, FM m) {
    constexpr int PK = pitch_k<DK>();
    frag_each(acc, m0, n0, [&](float &a, int t, int cc) {
        const float lt = Lg[t * PK + cc];
        float s = 0.f;
        for (int j = 0; j <= t; ++j) s = fmaf(m(t, j) * X[j * PK + cc], exp2f(lt - Lg[j * PK + cc]), s);
        a += s;
    });
}
template <int NT, int DK, typename FM>
__device__ __forceinline__ void gam_cols(float (&acc)[NT][4], int m0, int n0, const float *Lg,
                                         const float *X, FM m) {
    constexpr int PK = pitch_k<DK>();
    frag_each(acc, m0, n0, [&](float &a, int t, int cc) {
        const float lt = Lg[t * PK + cc];
        float s = 0.f;
        for (int u = t; u < kDC; ++u) s = fmaf(m(u, t) * X[u * PK + cc], exp2f(Lg[u * PK + cc] - lt), s);
        a += s;
    });
}

// Two fragment arrays of the same ownership, element by element.
template <int NT, typename F>
__device__ __forceinline__ void frag_each2(float (&d1)[NT][4], float (&d2)[NT][4], int m0, int n0, F f) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) f(d1[nt][r], d2[nt][r], m0 + g + 8 * (r >> 1), n0 + 8 * nt + 2 * t4 + (r & 1));
}

// part[h] holds a thread's share of row m0 + g + 8 h (summed over its columns): add the
// warp's row sums into buf (shared memory, several warps share a row).
__device__ __forceinline__ void rows_add(float (&part)[2], float *buf, int m0) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float s = part[h];
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        if ((lane & 3) == 0) atomicAdd(&buf[m0 + (lane >> 2) + 8 * h], s);
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
    constexpr bool SP = std::is_same<IO, float>::value;
    constexpr int PK = L::PK, NK = DK / 32;
    constexpr int DL = MODE == 3 ? DK : 1;   // entries of dL/dlam per token
    extern __shared__ float smem[];
    const ChunkTiles<MODE, DK> c(smem);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g8 = lane >> 2, t4 = lane & 3;
    const Own o = ownership<DK>();
    const int NS = DV / kDVS;
    const size_t bh = blockIdx.x / NS;
    const int j0 = (blockIdx.x % NS) * kDVS;
    const int nch = (T + kDC - 1) / kDC;
    const size_t row0 = bh * (size_t)T;

    constexpr bool kStage = L::kStage;
    constexpr int GW = MODE == 3 ? DK : 1;   // gate floats per token
    auto stage = [&](int chs) {
        const int ts = chs * kDC;
        stage_chunk(c, q, k, v, dO, gate, beta, states + ((bh * nch + chs) * DV + j0) * (size_t)DK, row0 + ts,
                    min(kDC, T - ts), DV, j0);
    };
    for (int p = tid; p < kDVS * DK; p += kDT)
        c.Hs[(p / DK) * PK + p % DK] = dST ? dST[(bh * DV + j0) * DK + p] : 0.f;
    if constexpr (kStage) stage(nch - 1);
    for (int ch = nch - 1; ch >= 0; --ch) {
        const int t0 = ch * kDC, n = min(kDC, T - t0), last = n - 1;
        const size_t rr = row0 + t0;
        if constexpr (kStage) {
            cp_async_wait_all();
            __syncthreads();
            unstage<kDT, IO>(c.sq, kDC, DK, n, c.Qs, PK);
            unstage<kDT, IO>(c.sk, kDC, DK, n, c.Ks, PK);
            unstage<kDT, IO>(c.sv, kDC, kDVS, n, c.Vs, kPV);
            unstage<kDT, IO>(c.sdo, kDC, kDVS, n, c.dOs, kPV);
            unstage<kDT, float>(c.sS, kDC, DK, kDVS, c.Ss, PK);
        } else {
            const float *src = states + ((bh * nch + ch) * DV + j0) * (size_t)DK;
            for (int p = tid; p < kDVS * DK; p += kDT) c.Ss[(p / DK) * PK + p % DK] = src[p];
            load_tile(q, rr, DK, 0, DK, n, c.Qs, PK);
            load_tile(k, rr, DK, 0, DK, n, c.Ks, PK);
            load_tile(v, rr, DV, j0, kDVS, n, c.Vs, kPV);
            load_tile(dO, rr, DV, j0, kDVS, n, c.dOs, kPV);
        }
        if (tid < DK) c.col1[tid] = 0.f;
        if (tid < kDC) c.dbl[tid] = c.dbs[tid] = c.dls[tid] = 0.f;
        __syncthreads();
        if (tid >= 32 && tid < 32 + DK) {   // colsum(S o H^T), while warp 0 scans the gates
            const int cc = tid - 32;
            float s = 0.f;
            for (int j = 0; j < kDVS; ++j) s = fmaf(c.Ss[j * PK + cc], c.Hs[j * PK + cc], s);
            c.col2[cc] = s;
        }
        if constexpr (kStage) {
            load_gates(c, gate ? c.sg : nullptr, c.sb, n, true);
            if (ch > 0) stage(ch - 1);   // the staging buffers have been read
        } else {
            load_gates(c, gate ? gate + rr * GW : nullptr, beta + rr, n, true);
        }
        grams<MODE, DK, SP>(c, true);
        __syncthreads();
        if (warp == 0) invert_unit_lower_32(c.Xm, c.Tm);
        __syncthreads();
        wy_factors<MODE, DK, SP>(c, true);   // W, U, dE = A^T dO + Kl H
        __syncthreads();
        new_values<MODE, DK, SP>(c);         // E = U - W S^T
        __syncthreads();

        {   // T^T dE (-> dv), dA = tril(dO E^T), dW = -dE S
            float td[1][4] = {}, da[1][4] = {}, dw[NK][4] = {};
            warp_mma<1, kDC, SP>(td, o.m0, o.n32, [&](int t, int u) { return c.Tm[u * kPC + t]; },
                                 [&](int u, int j) { return c.dEs[u * kPV + j]; });
            frag_each(td, o.m0, o.n32, [&](float &x, int t, int j) {
                c.TdE[t * kPV + j] = x;
                if (t < n) dv[(rr + t) * DV + j0 + j] = from_f32<IO>(c.bet[t] * x);
            });
            warp_mma<1, kDVS, SP>(da, o.m0, o.n32, [&](int t, int i) { return c.dOs[t * kPV + i]; },
                                  [&](int i, int j) { return c.Es[j * kPV + i]; });
            frag_each(da, o.m0, o.n32, [&](float &x, int t, int j) { c.dAm[t * kPC + j] = j <= t ? x : 0.f; });
            warp_mma<NK, kDVS, SP>(dw, o.m0, o.nk, [&](int t, int j) { return c.dEs[t * kPV + j]; },
                                   [&](int j, int cc) { return c.Ss[j * PK + cc]; });
            frag_each(dw, o.m0, o.nk, [&](float &x, int t, int cc) { c.dWm[t * PK + cc] = -x; });
        }
        __syncthreads();
        float tdw[NK][4] = {};
        {   // dT = dW (diag(b)Kg)^T + dE (diag(b)V)^T, strictly lower; T^T dW (held)
            float dt[1][4] = {};
            warp_mma<1, DK, SP>(dt, o.m0, o.n32, [&](int t, int cc) { return c.dWm[t * PK + cc]; },
                                [&](int cc, int u) { return c.kg(u, cc); });
            warp_mma<1, kDVS, SP>(dt, o.m0, o.n32, [&](int t, int j) { return c.dEs[t * kPV + j]; },
                                  [&](int j, int u) { return c.Vs[u * kPV + j]; });
            frag_each(dt, o.m0, o.n32,
                      [&](float &x, int t, int u) { c.dTm[t * kPC + u] = u < t ? c.bet[u] * x : 0.f; });
            warp_mma<NK, kDC, SP>(tdw, o.m0, o.nk, [&](int t, int u) { return c.Tm[u * kPC + t]; },
                                  [&](int u, int cc) { return c.dWm[u * PK + cc]; });
        }
        __syncthreads();
        {   // X = dT T^T (over Lm, no longer needed); T^T dW over dW
            float x[1][4] = {};
            warp_mma<1, kDC, SP>(x, o.m0, o.n32, [&](int t, int u) { return c.dTm[t * kPC + u]; },
                                 [&](int u, int j) { return c.Tm[j * kPC + u]; });
            frag_each(x, o.m0, o.n32, [&](float &val, int t, int j) { c.Xm[t * kPC + j] = val; });
            frag_each(tdw, o.m0, o.nk, [&](float &val, int t, int cc) { c.dWm[t * PK + cc] = val; });
        }
        __syncthreads();
        {   // dLm = -T^T X (strictly lower); BL = diag(b) dLm; mode 2 folds Gam into BL and dA
            float y[1][4] = {};
            warp_mma<1, kDC, SP>(y, o.m0, o.n32, [&](int t, int u) { return c.Tm[u * kPC + t]; },
                                 [&](int u, int j) { return c.Xm[u * kPC + j]; });
            float part[2] = {0.f, 0.f};
            frag_each(y, o.m0, o.n32, [&](float &val, int t, int j) {
                const float dlm = j < t ? -val : 0.f;
                part[(t - o.m0) >> 3] += dlm * c.Km[t * kPC + j];
                const float gm = MODE == 3 ? 1.f : c.Gm[t * kPC + j];
                c.BL[t * kPC + j] = c.bet[t] * dlm * gm;
                if (MODE != 3) c.dAm[t * kPC + j] *= gm;
            });
            rows_add(part, c.dbl, o.m0);
        }
        // (E H^T)-terms and the carried cotangent, both from H at the chunk's end
        float dkn[NK][4] = {}, hn[NK][4] = {};
        warp_mma<NK, kDVS, SP>(dkn, o.m0, o.nk, [&](int t, int j) { return c.Es[t * kPV + j]; },
                               [&](int j, int cc) { return c.Hs[j * PK + cc]; });
        frag_each(dkn, o.m0, o.nk, [&](float &x, int t, int cc) { x *= c.decf(t, cc, last); });
#pragma unroll
        for (int nt = 0; nt < NK; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {   // column sums of k o (g_L / g)(E H^T)
                const int cc = o.nk + 8 * nt + 2 * t4 + h;
                float s = fmaf(c.Ks[(o.m0 + g8) * PK + cc], dkn[nt][h],
                               c.Ks[(o.m0 + g8 + 8) * PK + cc] * dkn[nt][2 + h]);
                s += __shfl_xor_sync(0xffffffffu, s, 4);
                s += __shfl_xor_sync(0xffffffffu, s, 8);
                s += __shfl_xor_sync(0xffffffffu, s, 16);
                if (g8 == 0) atomicAdd(&c.col1[cc], s);
            }
        {   // dL/dS^T = Qg^T dO + diag(g_L) H - W^T dE  (rows j of this slice)
            float h2[NK][4] = {};
            warp_mma<NK, kDC, SP>(hn, o.m0, o.nk, [&](int j, int t) { return c.dOs[t * kPV + j]; },
                                  [&](int t, int cc) { return c.qg(t, cc); });
            warp_mma<NK, kDC, SP>(h2, o.m0, o.nk, [&](int j, int t) { return c.dEs[t * kPV + j]; },
                                  [&](int t, int cc) { return c.Wm[t * PK + cc]; });
            frag_each2(hn, h2, o.m0, o.nk, [&](float &x, float &y, int j, int cc) {
                x = fmaf(c.gl[cc], c.Hs[j * PK + cc], x - y);
            });
        }
        __syncthreads();
        frag_each(hn, o.m0, o.nk, [&](float &x, int j, int cc) { c.Hs[j * PK + cc] = x; });

        // dq, dk_plus, dk_minus
        float dq[NK][4] = {}, dkp[NK][4] = {};
        warp_mma<NK, kDVS, SP>(dq, o.m0, o.nk, [&](int t, int j) { return c.dOs[t * kPV + j]; },
                               [&](int j, int cc) { return c.Ss[j * PK + cc]; });
        frag_each2(dq, dkp, o.m0, o.nk, [&](float &x, float &y, int t, int cc) {
            const float gtc = c.gf(t, cc);
            x *= gtc;
            y = c.bet[t] * gtc * c.dWm[t * PK + cc];
        });
        if constexpr (MODE == 3) {
            gam_rows<NK, DK>(dq, o.m0, o.nk, c.Lg, c.Ks, [&](int t, int j) { return c.dAm[t * kPC + j]; });
            gam_rows<NK, DK>(dkp, o.m0, o.nk, c.Lg, c.Ks, [&](int t, int j) { return c.BL[t * kPC + j]; });
            gam_cols<NK, DK>(dkn, o.m0, o.nk, c.Lg, c.Qs, [&](int u, int t) { return c.dAm[u * kPC + t]; });
            gam_cols<NK, DK>(dkn, o.m0, o.nk, c.Lg, c.Ks, [&](int u, int t) { return c.BL[u * kPC + t]; });
        } else {
            warp_mma<NK, kDC, SP>(dq, o.m0, o.nk, [&](int t, int j) { return c.dAm[t * kPC + j]; },
                                  [&](int j, int cc) { return c.Ks[j * PK + cc]; });
            warp_mma<NK, kDC, SP>(dkp, o.m0, o.nk, [&](int t, int j) { return c.BL[t * kPC + j]; },
                                  [&](int j, int cc) { return c.Ks[j * PK + cc]; });
            warp_mma<NK, kDC, SP>(dkn, o.m0, o.nk, [&](int t, int u) { return c.dAm[u * kPC + t]; },
                                  [&](int u, int cc) { return c.Qs[u * PK + cc]; });
            warp_mma<NK, kDC, SP>(dkn, o.m0, o.nk, [&](int t, int u) { return c.BL[u * kPC + t]; },
                                  [&](int u, int cc) { return c.Ks[u * PK + cc]; });
        }
        __syncthreads();   // col1, col2 and dbl complete

        {   // this slice's shares of dq, dk, dL/dlam and db, into the fp32 accumulators
            float pdb[2] = {0.f, 0.f}, pdl[2] = {0.f, 0.f};
#pragma unroll
            for (int nt = 0; nt < NK; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {   // elements 2h, 2h+1: row t, columns cc, cc + 1
                    const int t = o.m0 + g8 + 8 * h, cc = o.nk + 8 * nt + 2 * t4;
                    float dl[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int r = 2 * h + e, ce = cc + e;
                        dl[e] = fmaf(c.Qs[t * PK + ce], dq[nt][r], c.Ks[t * PK + ce] * (dkp[nt][r] - dkn[nt][r]));
                        if (t == last) dl[e] += c.col1[ce] + c.gl[ce] * c.col2[ce];
                        pdb[h] = fmaf(c.kg(t, ce), c.dWm[t * PK + ce], pdb[h]);
                        pdl[h] += dl[e];
                    }
                    if (t < n) {
                        const size_t e0 = (rr + t) * DK + cc;
                        red_add2(dq_acc + e0, dq[nt][2 * h], dq[nt][2 * h + 1]);
                        red_add2(dk_acc + e0, dkp[nt][2 * h] + dkn[nt][2 * h], dkp[nt][2 * h + 1] + dkn[nt][2 * h + 1]);
                        if constexpr (DL > 1) red_add2(dl_acc + e0, dl[0], dl[1]);
                    }
                }
            rows_add(pdb, c.dbs, o.m0);
            if constexpr (DL == 1) rows_add(pdl, c.dls, o.m0);
        }
        __syncthreads();
        if (tid < n) {
            float p2 = 0.f;
            for (int j = 0; j < kDVS; ++j) p2 = fmaf(c.Vs[tid * kPV + j], c.TdE[tid * kPV + j], p2);
            atomicAdd(&db_acc[rr + tid], c.dbs[tid] + p2 + c.dbl[tid]);
            if constexpr (DL == 1) atomicAdd(&dl_acc[rr + tid], c.dls[tid]);
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

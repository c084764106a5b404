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
// The products are 32 x 32 to 128 x 128 tiles, each followed by an element-wise step: they
// run on the tensor cores as warp-level mma (bwd_util.cuh), with every computed operand
// split into high and low parts so that the products keep fp32 accuracy.
//
// fp32 I/O: one or two CTAs per (batch, head) (the d_k columns of S and G split between
// them): a forward sweep stores every chunk-start state in the caller's workspace, then a
// reverse sweep carries G back through the chunks and forms each chunk's gradients; a
// small kernel finishes dV and the gate gradient (m16n8k8 tf32 products).
//
// bf16 I/O: the two carries first (every S_c and G, one scan launch), then every chunk's
// gradients at once, then the gate gradient (m16n8k16 bf16 products; see below).
#include "la_internal.cuh"
#include "bwd_util.cuh"

#include <cfloat>
#include <type_traits>

namespace la {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kBwdC = 32;

// A head's d_k columns are split over SPLIT CTAs (2 at d_k = 128): each CTA owns DK/SPLIT
// columns of S and G, the products that stay within columns (dQ, dK, the state and G
// updates), and a share of those that sum over them (dV, dlam), which it adds into fp32
// accumulators in the workspace; a finishing kernel converts dV and takes the suffix sums.
// Row pitches are 4 (mod 32) floats (conflict-free mma operand loads).
template <int DK, int DV, int SPLIT>
struct BwdSmem {
    static constexpr int DKH = DK / SPLIT;
    static constexpr int PQ = DK + 4, PV = DV + 4, PS = DKH + 4, PC = kBwdC + 4;
    static constexpr int kQ = kBwdC * PQ, kV = kBwdC * PV, kS = DV * PS, kP = kBwdC * PC;
    // Qs Ks | Vs dOs | S, S_c, G | P dP | lam gv dec dl | red
    static constexpr int kFloats = 2 * kQ + 2 * kV + 3 * kS + 2 * kP + 4 * kBwdC + 8;
    static constexpr size_t kBytes = sizeof(float) * kFloats;
    static_assert(kBytes <= 227 * 1024, "shared memory");
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

// fragment coordinates of warp_mma's element r of n-tile nt (bwd_util.cuh)
__device__ __forceinline__ int frow(int m0, int r) { return m0 + ((threadIdx.x & 31) >> 2) + 8 * (r >> 1); }
__device__ __forceinline__ int fcol(int n0, int nt, int r) { return n0 + 8 * nt + 2 * (threadIdx.x & 3) + (r & 1); }

template <int DK, int DV, int SPLIT>
__global__ void __launch_bounds__(kBwdThreads)
backward_kernel(int T, int gate_heads, const float *__restrict__ q, const float *__restrict__ k,
                const float *__restrict__ v, const float *__restrict__ gate,
                const float *__restrict__ S0, const float *__restrict__ dO,
                const float *__restrict__ dST, float *__restrict__ dq, float *__restrict__ dk,
                float *__restrict__ dS0, float *__restrict__ ws, float *__restrict__ dv_acc,
                float *__restrict__ dl_acc) {
    // Operand splitting (bwd_util.cuh): every operand is split -- fp32 inputs have more
    // mantissa than tf32, and the gate gradient is a suffix sum over the whole sequence,
    // where one tf32 rounding per product adds up.
    constexpr bool SP = true;
    using L = BwdSmem<DK, DV, SPLIT>;
    constexpr int C = kBwdC, DKH = L::DKH, PQ = L::PQ, PV = L::PV, PS = L::PS, PC = L::PC;
    constexpr int NW = kBwdThreads / 32;
    // DV x DKH state tiles: DV / 16 row blocks of 16, the warps left over split the columns
    constexpr int RB = DV / 16, CG = NW / RB, NTS = DKH / 8 / CG;
    constexpr int NTQ = DKH / 32;             // C x DKH: rows 16 (w & 1), columns (DKH / 4)(w >> 1)
    constexpr int NTV = DV / 32;              // C x DV:  rows 16 (w & 1), columns (DV / 4)(w >> 1)
    static_assert(NW % RB == 0 && DKH % (8 * CG) == 0, "state partition");
    extern __shared__ float smem[];
    float *Qs = smem;                // [C][PQ]
    float *Ks = Qs + L::kQ;          // [C][PQ]
    float *Vs = Ks + L::kQ;          // [C][PV]
    float *dOs = Vs + L::kV;         // [C][PV]
    float *Sb0 = dOs + L::kV;        // [DV][PS]  chunk-start state (two buffers, reverse)
    float *Sb1 = Sb0 + L::kS;
    float *G = Sb1 + L::kS;          // [DV][PS]  dL/dS at the chunk's end
    float *P = G + L::kS;            // [C][PC]
    float *dP = P + L::kP;           // [C][PC]
    float *lam = dP + L::kP;         // [C]   in-chunk log-gate prefix
    float *gv = lam + C;             // [C]   g_t = exp(lam_t)
    float *dec = gv + C;             // [C]   g_L / g_t
    float *dl = dec + C;             // [C]   this CTA's share of dlam
    float *red = dl + C;             // [8]

    const int tid = threadIdx.x, warp = tid >> 5;
    const size_t bh = blockIdx.x / SPLIT;
    const int kh = blockIdx.x % SPLIT, c0 = kh * DKH;   // this CTA's columns c0 .. c0 + DKH
    const int nch = (T + C - 1) / C;
    const size_t row0 = bh * (size_t)T;
    const float *gh = gate ? (gate_heads ? gate + bh % gate_heads : gate + row0) : nullptr;
    const int gt = gate_heads ? 0 : 1;
    float *wsh = ws + (size_t)blockIdx.x * (nch + 1) * DV * DKH;
    const int mq = 16 * (warp & 1), n32 = 8 * (warp >> 1), nq = (DKH / 4) * (warp >> 1),
              nv = (DV / 4) * (warp >> 1);
    const int ms = 16 * (warp % RB), ns = (DKH / CG) * (warp / RB);

    // gates of chunk t0 (Lc tokens)
    auto load_gates = [&](int t0, int Lc) {
        if (warp == 0) {
            const int lane = tid & 31;
            float a = 1.f;
            if (gh && lane < Lc) a = gh[(size_t)(t0 + lane) * gt];
            float x = lane < Lc ? logf(fmaxf(a, FLT_MIN)) : 0.f;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += y;
            }
            const float xl = __shfl_sync(0xffffffffu, x, Lc - 1);
            lam[lane] = x;
            gv[lane] = expf(x);
            dec[lane] = expf(xl - x);
        }
    };
    auto load_direct = [&](const float *src, float *dst, int t0, int Lc, int d, int pitch) {
        for (int p = tid; p < C * d; p += kBwdThreads) {
            const int i = p / d, j = p % d;
            dst[i * pitch + j] = i < Lc ? src[(row0 + t0 + i) * d + j] : 0.f;
        }
    };

    // ---- forward sweep: chunk-start states (this CTA's columns) into the workspace
    float *S = Sb0;
    for (int p = tid; p < DV * DKH; p += kBwdThreads)
        S[(p / DKH) * PS + p % DKH] = S0 ? S0[bh * DV * DK + (p / DKH) * DK + c0 + p % DKH] : 0.f;
    __syncthreads();
    for (int c = 0; c <= nch; ++c) {
        for (int p = tid; p < DV * DKH / 4; p += kBwdThreads) {   // store S (float4)
            const int i = p / (DKH / 4), j = 4 * (p % (DKH / 4));
            *reinterpret_cast<float4 *>(wsh + (size_t)c * DV * DKH + i * DKH + j) =
                *reinterpret_cast<const float4 *>(S + i * PS + j);
        }
        if (c == nch) break;
        const int t0 = c * C, Lc = min(C, T - t0);
        load_direct(k, Ks, t0, Lc, DK, PQ);
        load_direct(v, Vs, t0, Lc, DV, PV);
        load_gates(t0, Lc);
        __syncthreads();
        // S <- g_L S + (dec o V)^T K   (this CTA's columns; state partition)
        const float gL = gv[Lc - 1];
        float acc[NTS][4] = {};
        warp_mma<NTS, C, true, SP>(acc, ms, ns, [&](int i, int j) { return dec[j] * Vs[j * PV + i]; },
                             [&](int j, int cc) { return Ks[j * PQ + c0 + cc]; });
#pragma unroll
        for (int nt = 0; nt < NTS; ++nt)
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                float &x = S[frow(ms, r) * PS + fcol(ns, nt, r)];
                x = fmaf(gL, x, acc[nt][r]);
            }
        __syncthreads();
    }

    // ---- reverse sweep
    // S holds this CTA's columns of S_T: its share of <dS_T, S_T> (dlam at the last token)
    float part0 = 0.f;
    for (int p = tid; p < DV * DKH; p += kBwdThreads) {
        const int i = p / DKH, j = p % DKH;
        const float g0 = dST ? dST[bh * DV * DK + i * DK + c0 + j] : 0.f;
        G[i * PS + j] = g0;
        part0 = fmaf(g0, S[i * PS + j], part0);
    }
    const float final_dot = block_sum(part0, red);
    if (tid == 0 && final_dot != 0.f) atomicAdd(&dl_acc[row0 + T - 1], final_dot);
    float *Sc = (S == Sb0) ? Sb1 : Sb0;   // the chunk's start state
    for (int c = nch - 1; c >= 0; --c) {
        const int t0 = c * C, Lc = min(C, T - t0);
        load_direct(q, Qs, t0, Lc, DK, PQ);
        load_direct(k, Ks, t0, Lc, DK, PQ);
        load_direct(v, Vs, t0, Lc, DV, PV);
        load_direct(dO, dOs, t0, Lc, DV, PV);
        const float *src = wsh + (size_t)c * DV * DKH;
        for (int p = tid; p < DV * DKH; p += kBwdThreads) Sc[(p / DKH) * PS + p % DKH] = src[p];
        if (tid < C) dl[tid] = 0.f;
        load_gates(t0, Lc);
        __syncthreads();
        {   // causal decayed score matrices P = (Q K^T) o D, dP = (dO V^T) o D
            float pp[1][4] = {}, dd[1][4] = {};
            warp_mma<1, DK, SP>(pp, mq, n32, [&](int t, int cc) { return Qs[t * PQ + cc]; },
                                [&](int cc, int j) { return Ks[j * PQ + cc]; });
            warp_mma<1, DV, SP>(dd, mq, n32, [&](int t, int i) { return dOs[t * PV + i]; },
                                [&](int i, int j) { return Vs[j * PV + i]; });
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int t = frow(mq, r), j = fcol(n32, 0, r);
                const float w = (t < Lc && j <= t) ? expf(lam[t] - lam[j]) : 0.f;
                P[t * PC + j] = pp[0][r] * w;
                dP[t * PC + j] = dd[0][r] * w;
            }
        }
        __syncthreads();
        {   // dQ = diag(g) dO S_c + dP K,  dK = dP^T Q + diag(g_L / g) V G  (this CTA's columns)
            float aq[NTQ][4] = {}, ak[NTQ][4] = {};
            warp_mma<NTQ, DV, SP, true>(aq, mq, nq, [&](int t, int i) { return dOs[t * PV + i]; },
                                  [&](int i, int cc) { return Sc[i * PS + cc]; });
            warp_mma<NTQ, DV, SP, true>(ak, mq, nq, [&](int t, int i) { return Vs[t * PV + i]; },
                                  [&](int i, int cc) { return G[i * PS + cc]; });
#pragma unroll
            for (int nt = 0; nt < NTQ; ++nt)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    aq[nt][r] *= gv[frow(mq, r)];
                    ak[nt][r] *= dec[frow(mq, r)];
                }
            warp_mma<NTQ, C, true, SP>(aq, mq, nq, [&](int t, int j) { return dP[t * PC + j]; },
                                 [&](int j, int cc) { return Ks[j * PQ + c0 + cc]; });
            warp_mma<NTQ, C, true, SP>(ak, mq, nq, [&](int t, int s2) { return dP[s2 * PC + t]; },
                                 [&](int s2, int cc) { return Qs[s2 * PQ + c0 + cc]; });
            float part[2] = {0.f, 0.f};
#pragma unroll
            for (int nt = 0; nt < NTQ; ++nt)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int t = frow(mq, r), cc = c0 + fcol(nq, nt, r);
                    part[r >> 1] += Qs[t * PQ + cc] * aq[nt][r] - Ks[t * PQ + cc] * ak[nt][r];
                    if (t < Lc) {
                        dq[(row0 + t0 + t) * DK + cc] = aq[nt][r];
                        dk[(row0 + t0 + t) * DK + cc] = ak[nt][r];
                    }
                }
#pragma unroll
            for (int h = 0; h < 2; ++h) {   // row sums of the warp into dl
                float s = part[h];
                s += __shfl_xor_sync(0xffffffffu, s, 1);
                s += __shfl_xor_sync(0xffffffffu, s, 2);
                if ((tid & 3) == 0) atomicAdd(&dl[mq + ((tid & 31) >> 2) + 8 * h], s);
            }
        }
        {   // dV = P^T dO + diag(g_L / g) K G^T: this CTA's columns' share, added up in fp32
            float av[NTV][4] = {};
            warp_mma<NTV, DKH, SP, true>(av, mq, nv, [&](int t, int cc) { return Ks[t * PQ + c0 + cc]; },
                                   [&](int cc, int i) { return G[i * PS + cc]; });
#pragma unroll
            for (int nt = 0; nt < NTV; ++nt)
#pragma unroll
                for (int r = 0; r < 4; ++r) av[nt][r] *= dec[frow(mq, r)];
            if (kh == 0)
                warp_mma<NTV, C, true, SP>(av, mq, nv, [&](int t, int s2) { return P[s2 * PC + t]; },
                                     [&](int s2, int i) { return dOs[s2 * PV + i]; });
#pragma unroll
            for (int nt = 0; nt < NTV; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int t = frow(mq, 2 * h), i = fcol(nv, nt, 2 * h);
                    if (t < Lc) {
                        float *dst = dv_acc + (row0 + t0 + t) * DV + i;
                        if (SPLIT == 1) *reinterpret_cast<float2 *>(dst) = make_float2(av[nt][2 * h], av[nt][2 * h + 1]);
                        else red_add2(dst, av[nt][2 * h], av[nt][2 * h + 1]);
                    }
                }
        }
        __syncthreads();   // dl complete; every read of G done
        if (tid < Lc) {
            if (SPLIT == 1) dl_acc[row0 + t0 + tid] += dl[tid];
            else atomicAdd(&dl_acc[row0 + t0 + tid], dl[tid]);
        }
        {   // carry G to the chunk start: G <- g_L G + dO^T diag(g) Q   (this CTA's columns)
            const float gL = gv[Lc - 1];
            float ag[NTS][4] = {};
            warp_mma<NTS, C, true, SP>(ag, ms, ns, [&](int i, int t) { return gv[t] * dOs[t * PV + i]; },
                                 [&](int t, int cc) { return Qs[t * PQ + c0 + cc]; });
#pragma unroll
            for (int nt = 0; nt < NTS; ++nt)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    float &x = G[frow(ms, r) * PS + fcol(ns, nt, r)];
                    x = fmaf(gL, x, ag[nt][r]);
                }
        }
        __syncthreads();
    }
    if (dS0)
        for (int p = tid; p < DV * DKH; p += kBwdThreads)
            dS0[bh * DV * DK + (p / DKH) * DK + c0 + p % DKH] = G[(p / DKH) * PS + p % DKH];
}

// ---------------------------------------------------------------------------------------
// bf16 I/O: every chunk's gradients at once.  The two carries are linear recurrences with
// no dependence on the gradients, so they run first, on their own:
//   (1) bwd_scan_kernel: S_c, the state at each chunk's start (forward from S_0), and G_c,
//       dL/dS at each chunk's end (backward from dS_T), into the workspace as bf16 high and
//       low planes (v = hi + lo to about 2^-17); one CTA per (b h, 32 rows of d_v, direction).
//   (2) bwd_chunk_kernel: one CTA per (b h, chunk): P, dP, dQ, dK, dV and the chunk's dlam
//       from S_c and G_c, every chunk in parallel.
//   (3) bwd_gate_kernel: <dS_T, S_T> at the last token and the suffix sums of dlam -> dgate.
// Every product is mma.sync m16n8k16 on bf16 tiles (fragments by ldmatrix, .trans for an
// operand stored transposed); q, k, v, dO are exact in bf16, and each computed operand
// (S, G, P, dP, the gate-weighted rows) enters as high and low parts (bwd_util.cuh), so the
// gate gradient's suffix sum over the sequence keeps fp32-level accuracy.
constexpr int kScanRows = 32;   // d_v rows of one scan CTA

// Workspace (bf16 I/O): per (b h) nch + 1 states S_c and nch cotangents G_c, each a
// [d_v][d_k] high plane then a low plane, then dlam [BH][T] fp32.
__host__ __device__ inline size_t bwd_plane_pairs(int BH, int nch) { return (size_t)BH * (2 * nch + 1); }

template <int DK>
struct ScanSmem {
    static constexpr int PK = DK + 8, PR = kScanRows + 8;            // bf16 pitches
    static constexpr int kB = kBwdC * PK, kA = kBwdC * PR;           // one buffer's B, A rows
    static constexpr int kO = kScanRows * PK;                         // one staged output plane
    static constexpr int kHalves = 2 * kB + 2 * kA + 2 * kA + 2 * kO; // buffers, Xh Xl, Oh Ol
    static constexpr size_t kBytes = 2 * (size_t)kHalves + 4 * (size_t)(5 * kBwdC);
};

// d_k / 32 warps; warp w owns columns 32w .. 32w + 31 of the CTA's 32 x d_k slice (two
// 16-row m-tiles, four 8-column n-tiles).  Direction 0: X = S, X_{c+1} = g_L X_c +
// (dec o V_c)^T K_c, X_c stored before each step and X_nch after the last.  Direction 1:
// X = G, X_{c-1} = g_L X_c + (g o dO_c)^T Q_c from X = dS_T, X_c stored before each step,
// the last X is dS_0.
template <int DK, int DV>
__global__ void __launch_bounds__(DK)
bwd_scan_kernel(int T, int gate_heads, const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ dO,
                const float *__restrict__ gate, const float *__restrict__ S0, const float *__restrict__ dST,
                float *__restrict__ dS0, __nv_bfloat16 *__restrict__ planes) {
    using L = ScanSmem<DK>;
    using bf = __nv_bfloat16;
    constexpr int C = kBwdC, PK = L::PK, PR = L::PR, NSL = DV / kScanRows, NTH = DK;
    extern __shared__ __align__(16) uint8_t ssm[];
    bf *Bt = reinterpret_cast<bf *>(ssm);     // [2][C][PK]   K or Q rows
    bf *At = Bt + 2 * L::kB;                  // [2][C][PR]   V or dO rows (this slice)
    bf *Xh = At + 2 * L::kA, *Xl = Xh + L::kA;
    bf *Oh = Xl + L::kA;                      // [2][kScanRows][PK]  X as high, low planes
    float *graw = reinterpret_cast<float *>(Oh + 2 * L::kO);   // [2][C]
    float *lam = graw + 2 * C, *wt = lam + C, *gL = wt + C;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sl = blockIdx.x % NSL, dir = (blockIdx.x / NSL) & 1;
    const size_t bh = blockIdx.x / NSL / 2;
    const int i0 = sl * kScanRows;
    const int nch = (T + C - 1) / C;
    const size_t row0 = bh * (size_t)T;
    const float *gh = gate ? (gate_heads ? gate + bh % gate_heads : gate + row0) : nullptr;
    const int gt = gate_heads ? 0 : 1;
    const bf *bsrc = dir ? q : k, *asrc = dir ? dO : v;
    const size_t plane = (size_t)DV * DK;
    bf *out = dir ? planes + 2 * plane * ((size_t)bh * nch + (size_t)gridDim.x / (2 * NSL) * (nch + 1))
                  : planes + 2 * plane * (bh * (size_t)(nch + 1));

    auto stage = [&](int c, int b) {
        const int t0 = c * C, Lc = min(C, T - t0);
        for (int p = tid; p < C * (DK / 8); p += NTH) {
            const int t = p / (DK / 8), x = 8 * (p % (DK / 8));
            bf *dst = Bt + b * L::kB + t * PK + x;
            if (t < Lc) cp_async16(dst, bsrc + (row0 + t0 + t) * DK + x);
            else *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
        }
        for (int p = tid; p < C * (kScanRows / 8); p += NTH) {
            const int t = p / (kScanRows / 8), x = 8 * (p % (kScanRows / 8));
            bf *dst = At + b * L::kA + t * PR + x;
            if (t < Lc) cp_async16(dst, asrc + (row0 + t0 + t) * DV + i0 + x);
            else *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
        }
        if (gh && gt && tid < Lc) cp_async4(graw + b * C + tid, gh + t0 + tid);
        cp_async_commit();
    };
    // this thread's accumulator elements: row i (of the slice), column cc
    auto arow = [&](int mt, int r) { return 16 * mt + (lane >> 2) + 8 * (r >> 1); };
    auto acol = [&](int nt, int r) { return 32 * warp + 8 * nt + 2 * (lane & 3) + (r & 1); };
    float acc[2][4][4];
    const float *init = dir ? dST : S0;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int r = 0; r < 4; ++r)
                acc[mt][nt][r] = init ? init[bh * plane + (size_t)(i0 + arow(mt, r)) * DK + acol(nt, r)] : 0.f;
    // X goes out through shared memory (high and low planes), then to state slot c in
    // 16-byte stores: the slice's rows are contiguous in each plane
    auto stash = [&]() {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int o = arow(mt, 2 * h) * PK + acol(nt, 2 * h);
                    const float x0 = acc[mt][nt][2 * h], x1 = acc[mt][nt][2 * h + 1];
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(x0, x1);
                    *reinterpret_cast<__nv_bfloat162 *>(Oh + o) = h2;
                    *reinterpret_cast<__nv_bfloat162 *>(Oh + L::kO + o) =
                        __floats2bfloat162_rn(x0 - __low2float(h2), x1 - __high2float(h2));
                }
    };
    auto flush = [&](int c) {
        bf *dst = out + 2 * plane * (size_t)c + (size_t)i0 * DK;
        for (int p = tid; p < 2 * kScanRows * (DK / 8); p += NTH) {
            const int pl = p / (kScanRows * (DK / 8)), r = p / (DK / 8) % kScanRows, x = 8 * (p % (DK / 8));
            *reinterpret_cast<uint4 *>(dst + pl * plane + (size_t)r * DK + x) =
                *reinterpret_cast<const uint4 *>(Oh + pl * L::kO + r * PK + x);
        }
    };
    int c = dir ? nch - 1 : 0;
    stage(c, 0);
    for (int it = 0; it < nch; ++it, c += dir ? -1 : 1) {
        const int b = it & 1, t0 = c * C, Lc = min(C, T - t0);
        stash();
        cp_async_wait_all();
        __syncthreads();   // chunk c and X staged; the previous step's reads of Xh, Xl done
        flush(c);
        if (it + 1 < nch) stage(dir ? c - 1 : c + 1, b ^ 1);
        if (warp == 0) {   // in-chunk log-gate prefix: dec_t = g_L / g_t (dir 0), g_t (dir 1)
            float a = 1.f;
            if (gh && lane < Lc) a = gt ? graw[b * C + lane] : gh[0];
            float x = lane < Lc ? logf(fmaxf(a, FLT_MIN)) : 0.f;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += y;
            }
            const float xl = __shfl_sync(0xffffffffu, x, Lc - 1);
            wt[lane] = expf(dir ? x : xl - x);
            if (lane == 0) gL[0] = expf(xl);
        }
        __syncthreads();
        for (int p = tid; p < C * kScanRows; p += NTH) {
            const int t = p / kScanRows, i = p % kScanRows;
            split_bf16(wt[t] * __bfloat162float(At[b * L::kA + t * PR + i]), Xh[t * PR + i], Xl[t * PR + i]);
        }
        __syncthreads();
        const float g = gL[0];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            float d[4][4] = {};
            mma_bf16_tiles<4, C, true, true>(d, 16 * mt, 32 * warp, Xh, Xl, PR, Bt + b * L::kB, nullptr, PK);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[mt][nt][r] = fmaf(g, acc[mt][nt][r], d[nt][r]);
        }
    }
    if (!dir) {
        stash();
        __syncthreads();
        flush(nch);
    } else if (dS0)
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int r = 0; r < 4; ++r)
                    dS0[bh * plane + (size_t)(i0 + arow(mt, r)) * DK + acol(nt, r)] = acc[mt][nt][r];
}

template <int DK, int DV>
struct ChunkSmem {
    static constexpr int PQ = DK + 8, PV = DV + 8, PC = kBwdC + 8;   // bf16 pitches
    // Q K | V dO | St (S_c, then G_c: high then low plane, [d_v][d_k] unpadded, swizzled) |
    // Ph Pl dPh dPl
    static constexpr int kSt = 2 * DV * DK;
    static constexpr int kHalves = 2 * kBwdC * PQ + 2 * kBwdC * PV + kSt + 4 * kBwdC * PC;
    static constexpr size_t kBytes = 2 * (size_t)kHalves + 4 * (size_t)(4 * kBwdC);
    static_assert(2 * kBwdC * PQ + kBwdC * PV <= kSt, "output staging");
};

// One CTA (8 warps) per (b h, chunk), two resident per SM: S_c and G_c pass through one
// tile in turn, G_c arriving while the S_c products finish.  P and dP: 16 x 8 blocks, warp w
// at rows 16 (w & 1), columns 8 (w >> 1); dQ, dK (C x d_k) and dV (C x d_v): rows 16 (w & 1),
// a quarter of the columns each.
template <int DK, int DV>
__global__ void __launch_bounds__(kBwdThreads, 2)
bwd_chunk_kernel(int T, int gate_heads, const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                 const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ dO,
                 const float *__restrict__ gate, const __nv_bfloat16 *__restrict__ planes,
                 __nv_bfloat16 *__restrict__ dq, __nv_bfloat16 *__restrict__ dk, __nv_bfloat16 *__restrict__ dv,
                 float *__restrict__ dl_out) {
    using L = ChunkSmem<DK, DV>;
    using bf = __nv_bfloat16;
    constexpr int C = kBwdC, PQ = L::PQ, PV = L::PV, PC = L::PC;
    constexpr int NTQ = DK / 32, NTV = DV / 32;
    extern __shared__ __align__(16) uint8_t csm[];
    bf *Qs = reinterpret_cast<bf *>(csm), *Ks = Qs + C * PQ, *Vs = Ks + C * PQ, *dOs = Vs + C * PV;
    bf *St = dOs + C * PV, *Stl = St + DV * DK;
    bf *Ph = St + L::kSt, *Pl = Ph + C * PC, *dPh = Pl + C * PC, *dPl = dPh + C * PC;
    float *lam = reinterpret_cast<float *>(dPl + C * PC), *gv = lam + C, *dec = gv + C, *dl = dec + C;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nch = (T + C - 1) / C;
    const size_t bh = blockIdx.x / nch;
    const int c = blockIdx.x % nch, t0 = c * C, Lc = min(C, T - t0);
    const size_t row0 = bh * (size_t)T, BH = gridDim.x / nch;
    const float *gh = gate ? (gate_heads ? gate + bh % gate_heads : gate + row0) : nullptr;
    const int gt = gate_heads ? 0 : 1;
    const size_t plane = (size_t)DV * DK;
    const bf *Sg = planes + 2 * plane * (bh * (nch + 1) + c);
    const bf *Gg = planes + 2 * plane * (BH * (nch + 1) + bh * nch + c);

    auto rows = [&](bf *dst, const bf *src, int d, int pitch) {
        for (int p = tid; p < C * (d / 8); p += kBwdThreads) {
            const int t = p / (d / 8), x = 8 * (p % (d / 8));
            if (t < Lc) cp_async16(dst + t * pitch + x, src + (row0 + t0 + t) * d + x);
            else *reinterpret_cast<uint4 *>(dst + t * pitch + x) = make_uint4(0u, 0u, 0u, 0u);
        }
    };
    auto state = [&](const bf *src) {   // high and low planes into St, 16-byte chunks swizzled by row
        for (int p = tid; p < 2 * DV * (DK / 8); p += kBwdThreads) {
            const int r = p / (DK / 8), j = p % (DK / 8);   // row r of [hi; lo]
            cp_async16(St + r * DK + 8 * (j ^ (r & 7)), src + (size_t)r * DK + 8 * j);
        }
        cp_async_commit();
    };
    if (warp == 0) {   // the chunk's log-gate prefix, while the other warps start the copies
        const float a = gh && lane < Lc ? gh[(size_t)(t0 + lane) * gt] : 1.f;
        float x = lane < Lc ? logf(fmaxf(a, FLT_MIN)) : 0.f;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        const float xl = __shfl_sync(0xffffffffu, x, Lc - 1);
        lam[lane] = x;
        gv[lane] = expf(x);
        dec[lane] = expf(xl - x);
        dl[lane] = 0.f;
    }
    rows(Qs, q, DK, PQ);
    rows(Ks, k, DK, PQ);
    rows(Vs, v, DV, PV);
    rows(dOs, dO, DV, PV);
    cp_async_commit();
    state(Sg);
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncthreads();   // inputs staged, gates ready
    const int mq = 16 * (warp & 1), n32 = 8 * (warp >> 1), nq = (DK / 4) * (warp >> 1), nv = (DV / 4) * (warp >> 1);
    {   // P = (Q K^T) o D, dP = (dO V^T) o D, as high and low parts
        float pp[1][4] = {}, dd[1][4] = {};
        mma_bf16_tiles<1, DK, false, false>(pp, mq, n32, Qs, nullptr, PQ, Ks, nullptr, PQ);
        mma_bf16_tiles<1, DV, false, false>(dd, mq, n32, dOs, nullptr, PV, Vs, nullptr, PV);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int t = mq + (lane >> 2) + 8 * (r >> 1), j = n32 + 2 * (lane & 3) + (r & 1);
            const float w = (t < Lc && j <= t) ? expf(lam[t] - lam[j]) : 0.f;
            split_bf16(pp[0][r] * w, Ph[t * PC + j], Pl[t * PC + j]);
            split_bf16(dd[0][r] * w, dPh[t * PC + j], dPl[t * PC + j]);
        }
    }
    cp_async_wait_all();
    __syncthreads();   // S_c staged; P, dP complete
    const int ra = mq + (lane >> 2), rb = ra + 8;   // this thread's fragment rows
    // dQ = diag(g) dO S_c + dP K
    float aq[NTQ][4] = {};
    mma_bf16_tiles<NTQ, DV, false, true, true>(aq, mq, nq, dOs, nullptr, PV, St, Stl, DK);
    __syncthreads();   // every read of S_c done: G_c takes its place
    state(Gg);
#pragma unroll
    for (int nt = 0; nt < NTQ; ++nt) aq[nt][0] *= gv[ra], aq[nt][1] *= gv[ra], aq[nt][2] *= gv[rb], aq[nt][3] *= gv[rb];
    mma_bf16_tiles<NTQ, C, false, true>(aq, mq, nq, dPh, dPl, PC, Ks, nullptr, PQ);
    float part[2] = {0.f, 0.f};
    auto dot = [&](const bf *X, float (&acc)[NTQ][4], float sg) {   // part[h] += sg X[t] . acc[t]
#pragma unroll
        for (int nt = 0; nt < NTQ; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int t = h ? rb : ra, cc = nq + 8 * nt + 2 * (lane & 3);
                const __nv_bfloat162 x2 = *reinterpret_cast<const __nv_bfloat162 *>(X + t * PQ + cc);
                part[h] += sg * (__low2float(x2) * acc[nt][2 * h] + __high2float(x2) * acc[nt][2 * h + 1]);
            }
    };
    dot(Qs, aq, 1.f);
    cp_async_wait_all();
    __syncthreads();   // G_c staged
    // dK = diag(g_L / g) V G + dP^T Q;  dV = diag(g_L / g) K G^T + P^T dO
    float ak[NTQ][4] = {}, av[NTV][4] = {};
    mma_bf16_tiles<NTQ, DV, false, true, true>(ak, mq, nq, Vs, nullptr, PV, St, Stl, DK);
    mma_bf16_tiles<NTV, DK, false, false, true>(av, mq, nv, Ks, nullptr, PQ, St, Stl, DK);
    const float ea = dec[ra], eb = dec[rb];
#pragma unroll
    for (int nt = 0; nt < NTQ; ++nt) ak[nt][0] *= ea, ak[nt][1] *= ea, ak[nt][2] *= eb, ak[nt][3] *= eb;
#pragma unroll
    for (int nt = 0; nt < NTV; ++nt) av[nt][0] *= ea, av[nt][1] *= ea, av[nt][2] *= eb, av[nt][3] *= eb;
    mma_bf16_tiles<NTQ, C, true, true>(ak, mq, nq, dPh, dPl, PC, Qs, nullptr, PQ);
    mma_bf16_tiles<NTV, C, true, true>(av, mq, nv, Ph, Pl, PC, dOs, nullptr, PV);
    dot(Ks, ak, -1.f);
#pragma unroll
    for (int h = 0; h < 2; ++h) {   // dlam_t = q_t . dq_t - k_t . dk_t: the warp's row sums
        float s = part[h];
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        if ((lane & 3) == 0) atomicAdd(&dl[h ? rb : ra], s);
    }
    __syncthreads();   // every read of G_c done: the tile takes the outputs
    bf *Oq = St, *Ok = Oq + C * PQ, *Ov = Ok + C * PQ;   // [C][PQ] [C][PQ] [C][PV]
    auto put = [&](bf *O, int pitch, int n0, int i, float (&acc)[4]) {
        *reinterpret_cast<__nv_bfloat162 *>(O + ra * pitch + n0 + i) = __floats2bfloat162_rn(acc[0], acc[1]);
        *reinterpret_cast<__nv_bfloat162 *>(O + rb * pitch + n0 + i) = __floats2bfloat162_rn(acc[2], acc[3]);
    };
#pragma unroll
    for (int nt = 0; nt < NTQ; ++nt) {
        put(Oq, PQ, nq + 8 * nt, 2 * (lane & 3), aq[nt]);
        put(Ok, PQ, nq + 8 * nt, 2 * (lane & 3), ak[nt]);
    }
#pragma unroll
    for (int nt = 0; nt < NTV; ++nt) put(Ov, PV, nv + 8 * nt, 2 * (lane & 3), av[nt]);
    __syncthreads();
    auto out_rows = [&](bf *dst, const bf *src, int d, int pitch) {   // rows t < Lc, 16-byte stores
        for (int p = tid; p < Lc * (d / 8); p += kBwdThreads) {
            const int t = p / (d / 8), x = 8 * (p % (d / 8));
            *reinterpret_cast<uint4 *>(dst + (row0 + t0 + t) * d + x) = *reinterpret_cast<const uint4 *>(src + t * pitch + x);
        }
    };
    out_rows(dq, Oq, DK, PQ);
    out_rows(dk, Ok, DK, PQ);
    out_rows(dv, Ov, DV, PV);
    if (tid < Lc) dl_out[row0 + t0 + tid] = dl[tid];
}

// Per (b h): dlam at the last token gains <dS_T, S_T> (S_T the last stored state, high + low
// planes); then d log a_t = sum_{u >= t} dlam_u, da_t = d log a_t / a_t.
__global__ void __launch_bounds__(kBwdThreads)
bwd_gate_kernel(int T, int DK, int DV, const float *__restrict__ dST, const __nv_bfloat16 *__restrict__ planes,
                const float *__restrict__ dl, const float *__restrict__ gate, float *__restrict__ dgate) {
    __shared__ float tot[kBwdThreads];
    __shared__ float red[kBwdThreads / 32];
    const size_t bh = blockIdx.x, row0 = bh * (size_t)T;
    const int tid = threadIdx.x, nch = (T + kBwdC - 1) / kBwdC;
    const size_t plane = (size_t)DV * DK;
    float last = 0.f;
    if (dST) {
        const __nv_bfloat16 *hi = planes + 2 * plane * (bh * (nch + 1) + nch), *lo = hi + plane;
        float s = 0.f;
        for (size_t e = tid; e < plane; e += kBwdThreads)
            s = fmaf(dST[bh * plane + e], __bfloat162float(hi[e]) + __bfloat162float(lo[e]), s);
        last = block_sum(s, red);
    }
    const int per = (T + kBwdThreads - 1) / kBwdThreads;
    const int a0 = min(T, tid * per), a1 = min(T, a0 + per);
    float s = 0.f;
    for (int t = a0; t < a1; ++t) s += dl[row0 + t];
    if (a0 <= T - 1 && T - 1 < a1) s += last;
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
        run += dl[row0 + t] + (t == T - 1 ? last : 0.f);
        dgate[row0 + t] = run / fmaxf(gate[row0 + t], FLT_MIN);
    }
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
    const size_t nch = ((size_t)T + kBwdC - 1) / kBwdC;
    cudaError_t e;
    if constexpr (std::is_same<IO, __nv_bfloat16>::value) {
        using bf = __nv_bfloat16;
        const bf *qb = static_cast<const bf *>(q), *kb = static_cast<const bf *>(k),
                 *vb = static_cast<const bf *>(v), *db = static_cast<const bf *>(dO);
        bf *planes = reinterpret_cast<bf *>(ws);
        float *dl = ws + bwd_plane_pairs(BH, (int)nch) * DV * DK;
        auto scan = bwd_scan_kernel<DK, DV>;
        auto chunk = bwd_chunk_kernel<DK, DV>;
        e = cudaFuncSetAttribute(chunk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ChunkSmem<DK, DV>::kBytes);
        if (e == cudaSuccess)   // two CTAs per SM
            e = cudaFuncSetAttribute(chunk, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) return e;
        timer_begin(st);
        scan<<<(unsigned)(BH * 2 * (DV / kScanRows)), DK, ScanSmem<DK>::kBytes, st>>>(
            T, gate_heads, qb, kb, vb, db, gate, S0, dST, dS0, planes);
        timer_end(st);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        timer_begin(st);
        chunk<<<(unsigned)(BH * nch), kBwdThreads, ChunkSmem<DK, DV>::kBytes, st>>>(
            T, gate_heads, qb, kb, vb, db, gate, planes, static_cast<bf *>(dq), static_cast<bf *>(dk),
            static_cast<bf *>(dv), dl);
        timer_end(st);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if (dgate) {
            timer_begin(st);
            bwd_gate_kernel<<<(unsigned)BH, kBwdThreads, 0, st>>>(T, DK, DV, dST, planes, dl, gate, dgate);
            timer_end(st);
        }
        note_launches(dgate ? 3 : 2);
        return cudaGetLastError();
    } else {
        constexpr int SPLIT = bwd_split<DK>();
        using L = BwdSmem<DK, DV, SPLIT>;
        float *dv_acc = ws + (size_t)BH * (nch + 1) * DV * DK;
        float *dl_acc = dv_acc + (size_t)BH * T * DV;
        e = cudaMemsetAsync(dv_acc, 0, sizeof(float) * (size_t)BH * T * (DV + 1), st);
        if (e != cudaSuccess) return e;
        auto kern = backward_kernel<DK, DV, SPLIT>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kBytes);
        if (e != cudaSuccess) return e;
        timer_begin(st);
        kern<<<(unsigned)(BH * SPLIT), kBwdThreads, L::kBytes, st>>>(
            T, gate_heads, static_cast<const float *>(q), static_cast<const float *>(k), static_cast<const float *>(v),
            gate, S0, static_cast<const float *>(dO), dST, static_cast<float *>(dq), static_cast<float *>(dk), dS0,
            ws, dv_acc, dl_acc);
        timer_end(st);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        timer_begin(st);
        backward_finish_kernel<IO><<<(unsigned)BH, kBwdThreads, 0, st>>>(
            T, DV, dv_acc, static_cast<IO *>(dv), dl_acc, gate, dgate);
        timer_end(st);
        note_launches(2);
        return cudaGetLastError();
    }
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
    // bf16 I/O: every chunk-start state and chunk-end cotangent (bf16 high and low planes),
    // then dlam; fp32 I/O: every chunk-start state, then the fp32 accumulators of dv and
    // dlam.  The first is never the smaller (nch d_k >= 2 T).
    return sizeof(float) * (size_t)B * H * ((2 * nch + 1) * d_k * d_v + (size_t)T);
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
    if (BH * 2 * (d_v / kScanRows) > INT32_MAX) return LA_ERR_INVALID_ARG;   // the scan's grid
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

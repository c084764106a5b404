// prefill_simt.cu -- chunked prefill on CUDA cores, fp32 arithmetic throughout.
//
// This is the kernel for fp32 I/O (where a bf16 tensor-core product could not hold the
// fp32 tolerance) and for the d = 64 shapes.  It evaluates the chunked form of "Linear
// attention and hybrids", section "Three forms of one computation": inside a chunk of C
// tokens the causally masked C x C matrix, across chunks the state carried in shared
// memory.  With L tokens in the chunk, in-chunk log-gate prefix lam_i = sum_{m<=i} log a_m
// (so the page's decay-mask entry D_ij = a_{j+1}...a_i is exp(lam_i - lam_j), section
// "Memory must forget"), g_i = exp(lam_i), and X the chunk's value rows:
//
//   A_ij = (q_i . k_j) exp(lam_i - lam_j)  for j <= i   (phi(q), phi(k) in mode 0)
//   O    = diag(g) Q S^T + A X              (mode 0: divided by den_i = sum_j A_ij + q_i.z)
//   S   <- g_L S + sum_j exp(lam_L - lam_j) x_j k_j^T,   z <- z + sum_j phi(k_j)
//
// Modes 0/1 use X = V.  Mode 2 (the Gated DeltaNet update of section "The delta rule and
// Gated DeltaNet") replaces V by the write vectors e_t = b_t (v_t - a_t S_{t-1} k_t),
// which solve a unit lower-triangular system inside the chunk:
//
//   (I + Lm) E = diag(b) V - diag(b g) K S^T,   Lm_ij = b_i exp(lam_i - lam_j) (k_i . k_j), j < i
//
// solved here by forward substitution as U = (I+Lm)^-1 diag(b) V, W = (I+Lm)^-1 diag(b g) K,
// E = U - W S^T.  Every exponent is <= 0, so no factor exceeds 1.
//
// Mode 3 (Kimi Delta Attention, the same section: Diag(a_t) in place of the scalar a_t,
// one decay per channel c of d_k) takes the in-chunk prefix per channel, lam_ic, and
// the decay of key j seen from row i becomes exp(lam_ic - lam_jc) inside the dot products:
//
//   A_ij = sum_c q_ic k_jc exp(lam_ic - lam_jc),  Lm_ij = b_i sum_c k_ic k_jc exp(lam_ic - lam_jc),
//   (I + Lm) E = diag(b) V - diag(b) (K o G) S^T,   G_ic = exp(lam_ic),
//   O = (Q o G) S^T + A E,   S <- S Diag(G_L) + E^T (K o exp(lam_L - lam)).
//
// One CTA (256 threads) per (batch, head) -- or per (sequence, head) of packed
// variable-length sequences -- walks the chunks in order; all tiles are fp32 in shared
// memory.  The chunk's products (Q K^T, K K^T, W S^T, Q S^T, A X and the state update)
// run on the tensor cores as warp-level mma (tf32 m16n8k8, each operand split into a tf32
// part and its remainder: three products per tile, fp32 accuracy), in 16 x 32 tiles dealt
// round-robin to the eight warps; row pitches are 4 (mod 32) floats so that the fragment
// loads are conflict free.  Mode 3's A and Lm keep a per-term exponential inside the dot
// product and stay on the CUDA cores (there the pitch is d + 1, conflict free for its
// row-strided reads); the forward substitution is a CUDA-core recurrence in every mode.
#include "la_internal.cuh"
#include "bwd_util.cuh"

#include <cfloat>

namespace la {
namespace {

constexpr int kSimtThreads = 256;

template <int MODE, int DK, int DV, int C>
struct SimtSmem {
    static constexpr int SK = DK + (MODE == 3 ? 1 : 4), SV = DV + 4, SA = C + 4;   // row pitches
    static constexpr int kS = DV * SK;
    static constexpr int kQ = C * SK;
    static constexpr int kV = C * SV;
    static constexpr int kA = C * SA;
    static constexpr int kLamC = (MODE == 3) ? kQ : 0;   // per-channel log-gate prefix
    static constexpr int kFloats = kS + 3 * kQ + kV + 2 * kA + 4 * C + DK + kLamC;
    static constexpr int kRawOff = (kFloats + 3) & ~3;   // 16-byte aligned: the next chunk's raw rows
    template <typename IO>
    static constexpr size_t bytes() { return sizeof(float) * kRawOff + sizeof(IO) * (2 * C * DK + C * DV); }
};

template <int MODE, int DK, int DV, int C, typename IO>
__global__ void __launch_bounds__(kSimtThreads)
prefill_simt_kernel(int T, int H, const int *__restrict__ cu, const IO *__restrict__ q,
                    const IO *__restrict__ k, const IO *__restrict__ v,
                    const float *__restrict__ gate, const float *__restrict__ beta,
                    float *__restrict__ state, float *__restrict__ zg, IO *__restrict__ o,
                    int init_state, unsigned *err, int gate_heads) {
    using L = SimtSmem<MODE, DK, DV, C>;
    constexpr bool kDelta = (MODE == 2 || MODE == 3);
    extern __shared__ float smem[];
    float *S = smem;                 // [DV][DK+1]
    float *Qs = S + L::kS;           // [C][DK+1]
    float *Ks = Qs + L::kQ;          // [C][DK+1]
    float *Ws = Ks + L::kQ;          // [C][DK+1]  mode 2
    float *Vs = Ws + L::kQ;          // [C][DV+1]  V, then U, then E in mode 2
    float *A = Vs + L::kV;           // [C][C+1]
    float *Lm = A + L::kA;           // [C][C+1]   mode 2
    float *lam = Lm + L::kA;         // [C]
    float *bet = lam + C;            // [C]
    float *den = bet + C;            // [C]
    float *dec = den + C;            // [C]
    float *zs = dec + C;             // [DK]
    float *lamC = zs + DK;           // [C][DK+1]  mode 3
    IO *Rq = reinterpret_cast<IO *>(smem + L::kRawOff);   // raw q, k, v rows of the next chunk
    IO *Rk = Rq + C * DK;
    IO *Rv = Rk + C * DK;

    constexpr int SK = L::SK, SV = L::SV, SA = L::SA;
    const int tid = threadIdx.x, lane = tid & 31;
    // the warp's 16 x 32 tiles of an M x N product (four 8-column n-tiles), round-robin
    auto for_tiles = [&](int M, int N, auto f) {
        const int per = N / 32, ntile = (M / 16) * per;
        for (int mt = tid >> 5; mt < ntile; mt += kSimtThreads / 32) f(16 * (mt / per), 32 * (mt % per));
    };
    // fragment element r of n-tile nt at (m0, n0): row, column
    auto frow = [&](int m0, int r) { return m0 + (lane >> 2) + 8 * (r >> 1); };
    auto fcol = [&](int n0, int nt, int r) { return n0 + 8 * nt + 2 * (lane & 3) + (r & 1); };
    // The state slot is blockIdx.x: (batch, head) for dense tensors, (sequence, head) for
    // packed ones.  row0 is the first token row of the CTA in the [rows][d] view of
    // q, k, v and o, n its token count.
    const size_t bh = blockIdx.x;
    size_t row0 = bh * (size_t)T;
    int n = T;
    if (cu) {   // packed: sequence blockIdx.x / H of head row blockIdx.x % H
        const int sq = blockIdx.x / H, hr = blockIdx.x % H;
        const int a = cu[sq], b = cu[sq + 1];
        const int tb = min(max(a, 0), T), te = min(max(b, tb), T);
        if ((a != tb || b != te) && tid == 0 && err) atomicOr(err, (unsigned)kErrBadInput);
        row0 = (size_t)hr * T + tb;
        n = te - tb;
    }
    const IO *qh = q + row0 * DK;
    const IO *kh = k + row0 * DK;
    const IO *vh = v + row0 * DV;
    IO *oh = o + row0 * DV;
    // per-token gates from row0 on, or (gate_heads > 0) one constant gate for the head
    const float *gh = gate ? (gate_heads ? gate + blockIdx.x % gate_heads : gate + row0 * (MODE == 3 ? DK : 1))
                           : nullptr;
    const int gt = gate_heads ? 0 : 1;   // token stride of gh (modes 1, 2)
    const float *bh_beta = beta ? beta + row0 : nullptr;
    float *Sg = state + bh * (size_t)DV * DK;

    // the raw q, k, v rows [t0, t0 + C) of the CTA's tokens into Rq, Rk, Rv (16-byte copies,
    // in flight while the previous chunk is processed; rows past the end are not copied)
    auto issue_raw = [&](int t0) {
        const int Lc = min(C, n - t0);
        constexpr int QK16 = DK * (int)sizeof(IO) / 16, V16 = DV * (int)sizeof(IO) / 16;
        for (int p = tid; p < Lc * QK16; p += kSimtThreads) {
            const int i = p / QK16, x = p % QK16;
            cp_async16(reinterpret_cast<uint8_t *>(Rq + i * DK) + 16 * x,
                       reinterpret_cast<const uint8_t *>(qh + (size_t)(t0 + i) * DK) + 16 * x);
            cp_async16(reinterpret_cast<uint8_t *>(Rk + i * DK) + 16 * x,
                       reinterpret_cast<const uint8_t *>(kh + (size_t)(t0 + i) * DK) + 16 * x);
        }
        for (int p = tid; p < Lc * V16; p += kSimtThreads) {
            const int i = p / V16, x = p % V16;
            cp_async16(reinterpret_cast<uint8_t *>(Rv + i * DV) + 16 * x,
                       reinterpret_cast<const uint8_t *>(vh + (size_t)(t0 + i) * DV) + 16 * x);
        }
        cp_async_commit();
    };
    if (n > 0) issue_raw(0);
    for (int p = tid; p < DV * DK; p += kSimtThreads)
        S[(p / DK) * SK + p % DK] = init_state ? Sg[p] : 0.f;
    if (MODE == 0)
        for (int p = tid; p < DK; p += kSimtThreads) zs[p] = init_state ? zg[bh * DK + p] : 0.f;

    for (int t0 = 0; t0 < n; t0 += C) {
        const int Lc = min(C, n - t0);
        cp_async_wait_all();
        __syncthreads();   // the chunk's raw rows are in (and the previous chunk is done)
        // ---- the chunk's tiles from the raw rows (phi applied in mode 0) and the gates
        for (int p = tid; p < C * DK; p += kSimtThreads) {   // rows past the chunk's end: zero
            const int i = p / DK, j = p % DK;
            float qv = 0.f, kv = 0.f;
            if (i < Lc) {
                qv = to_f32(Rq[i * DK + j]);
                kv = to_f32(Rk[i * DK + j]);
                if (MODE == 0) { qv = feature_phi(qv); kv = feature_phi(kv); }
            }
            Qs[i * SK + j] = qv;
            Ks[i * SK + j] = kv;
            if (kDelta) Ws[i * SK + j] = 0.f;
        }
        for (int p = tid; p < C * DV; p += kSimtThreads)
            Vs[(p / DV) * SV + p % DV] = p / DV < Lc ? to_f32(Rv[(p / DV) * DV + p % DV]) : 0.f;
        if (tid < Lc) {
            lam[tid] = (MODE != 0 && MODE != 3 && gh) ? logf(fmaxf(gh[(t0 + tid) * gt], FLT_MIN)) : 0.f;
            bet[tid] = kDelta ? bh_beta[t0 + tid] : 0.f;
        }
        if (MODE == 3) {   // per-channel in-chunk prefix of log a, one channel per thread
            for (int c = tid; c < DK; c += kSimtThreads) {
                float acc = 0.f;
                for (int i = 0; i < Lc; ++i) {
                    acc += gh ? logf(fmaxf(gh[(size_t)(t0 + i) * DK + c], FLT_MIN)) : 0.f;
                    lamC[i * SK + c] = acc;
                }
            }
        }
        __syncthreads();   // the raw rows are read: the next chunk's may land
        if (t0 + C < n) issue_raw(t0 + C);
        if (tid == 0)
            for (int i = 1; i < Lc; ++i) lam[i] += lam[i - 1];
        __syncthreads();
        if (tid < Lc) dec[tid] = expf(lam[Lc - 1] - lam[tid]);

        // ---- intra-chunk scores A (and the delta-rule matrix Lm)
        if constexpr (MODE == 3) {   // a decay per channel inside the dot products
            for (int p = tid; p < C * C; p += kSimtThreads) {
                const int i = p / C, j = p % C;
                float aij = 0.f, lij = 0.f;
                if (i < Lc && j <= i) {
                    float qk = 0.f, kk = 0.f;
#pragma unroll 8
                    for (int c = 0; c < DK; ++c) {
                        const float kj = Ks[j * SK + c] * expf(lamC[i * SK + c] - lamC[j * SK + c]);
                        qk = fmaf(Qs[i * SK + c], kj, qk);
                        kk = fmaf(Ks[i * SK + c], kj, kk);
                    }
                    aij = qk;
                    if (j < i) lij = bet[i] * kk;
                }
                A[i * SA + j] = aij;
                Lm[i * SA + j] = lij;
            }
        } else {
            for_tiles(C, C, [&](int m0, int n0) {
                float qk[4][4] = {}, kk[4][4] = {};
                warp_mma<4, DK, true>(qk, m0, n0, [&](int i, int c) { return Qs[i * SK + c]; },
                                      [&](int c, int j) { return Ks[j * SK + c]; });
                if (kDelta)
                    warp_mma<4, DK, true>(kk, m0, n0, [&](int i, int c) { return Ks[i * SK + c]; },
                                          [&](int c, int j) { return Ks[j * SK + c]; });
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int i = frow(m0, r), j = fcol(n0, nt, r);
                        const bool in = i < Lc && j <= i;
                        const float d = (MODE == 0 || !in) ? 1.f : expf(lam[i] - lam[j]);
                        A[i * SA + j] = in ? qk[nt][r] * d : 0.f;
                        if (kDelta) Lm[i * SA + j] = (in && j < i) ? bet[i] * d * kk[nt][r] : 0.f;
                    }
            });
        }
        __syncthreads();

        if (MODE == 0 && tid < Lc) {
            float s = 0.f;
            for (int j = 0; j <= tid; ++j) s += A[tid * SA + j];
            for (int c = 0; c < DK; ++c) s = fmaf(Qs[tid * SK + c], zs[c], s);
            den[tid] = s;
        }

        if (kDelta) {
            // right-hand sides: diag(b) V in Vs, diag(b g) K (mode 3: diag(b) (K o G)) in Ws
            for (int p = tid; p < Lc * DV; p += kSimtThreads) Vs[(p / DV) * SV + p % DV] *= bet[p / DV];
            for (int p = tid; p < Lc * DK; p += kSimtThreads) {
                const int i = p / DK, c = p % DK;
                const float g = (MODE == 3) ? expf(lamC[i * SK + c]) : expf(lam[i]);
                Ws[i * SK + c] = bet[i] * g * Ks[i * SK + c];
            }
            __syncthreads();
            // forward substitution, one column of [U | W] per thread
            for (int r = 1; r < Lc; ++r) {
                for (int col = tid; col < DV + DK; col += kSimtThreads) {
                    float *X = col < DV ? Vs + col : Ws + (col - DV);
                    const int stride = col < DV ? SV : SK;
                    float acc = X[r * stride];
                    for (int j = 0; j < r; ++j) acc = fmaf(-Lm[r * SA + j], X[j * stride], acc);
                    X[r * stride] = acc;
                }
                __syncthreads();
            }
            // E = U - W S^T, in place over U (rows past the chunk's end stay zero)
            for_tiles(C, DV, [&](int m0, int n0) {
                float ws[4][4] = {};
                warp_mma<4, DK, true>(ws, m0, n0, [&](int t, int c) { return Ws[t * SK + c]; },
                                      [&](int c, int i) { return S[i * SK + c]; });
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int t = frow(m0, r), i = fcol(n0, nt, r);
                        Vs[t * SV + i] = t < Lc ? Vs[t * SV + i] - ws[nt][r] : 0.f;
                    }
            });
        }
        __syncthreads();
        if (MODE == 3) {
            // Q <- Q o G (the inter-chunk read) and K <- K o exp(lam_L - lam) (the state
            // update); the raw tiles are no longer needed
            for (int p = tid; p < Lc * DK; p += kSimtThreads) {
                const int i = p / DK, c = p % DK;
                Qs[i * SK + c] *= expf(lamC[i * SK + c]);
                Ks[i * SK + c] *= expf(lamC[(Lc - 1) * SK + c] - lamC[i * SK + c]);
            }
            __syncthreads();
        }

        // ---- output: O = diag(g) Q S^T + A X   (mode 0: / den)
        for_tiles(C, DV, [&](int m0, int n0) {
            float inter[4][4] = {}, intra[4][4] = {};
            warp_mma<4, DK, true>(inter, m0, n0, [&](int t, int c) { return Qs[t * SK + c]; },
                                  [&](int c, int i) { return S[i * SK + c]; });
            warp_mma<4, C, true>(intra, m0, n0, [&](int t, int j) { return A[t * SA + j]; },
                                 [&](int j, int i) { return Vs[j * SV + i]; });
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int t = frow(m0, r), i = fcol(n0, nt, r);
                    if (t >= Lc) continue;
                    float out;
                    if (MODE == 0) out = (inter[nt][r] + intra[nt][r]) / den[t];
                    else if (MODE == 3) out = inter[nt][r] + intra[nt][r];
                    else out = fmaf(expf(lam[t]), inter[nt][r], intra[nt][r]);
                    oh[(size_t)(t0 + t) * DV + i] = from_f32<IO>(out);
                }
        });
        __syncthreads();

        // ---- state update: S <- g_L S + sum_j exp(lam_L - lam_j) x_j k_j^T
        const float gL = (MODE == 0 || MODE == 3) ? 1.f : expf(lam[Lc - 1]);
        for_tiles(DV, DK, [&](int m0, int n0) {
            float acc[4][4] = {};
            warp_mma<4, C, true>(acc, m0, n0,
                                 [&](int i, int j) { return j < Lc ? (MODE == 3 ? 1.f : dec[j]) * Vs[j * SV + i] : 0.f; },
                                 [&](int j, int c) { return Ks[j * SK + c]; });
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int i = frow(m0, r), c = fcol(n0, nt, r);
                    const float g = (MODE == 3) ? expf(lamC[(Lc - 1) * SK + c]) : gL;
                    S[i * SK + c] = fmaf(g, S[i * SK + c], acc[nt][r]);
                }
        });
        if (MODE == 0) {
            for (int c = tid; c < DK; c += kSimtThreads) {
                float acc = 0.f;
                for (int j = 0; j < Lc; ++j) acc += Ks[j * SK + c];
                zs[c] += acc;
            }
        }
        __syncthreads();
    }

    for (int p = tid; p < DV * DK; p += kSimtThreads) Sg[p] = S[(p / DK) * SK + p % DK];
    if (MODE == 0)
        for (int p = tid; p < DK; p += kSimtThreads) zg[bh * DK + p] = zs[p];
}

template <int MODE, int DK, int DV, int C, typename IO>
cudaError_t launch_one(const PrefillArgs &a) {
    using L = SimtSmem<MODE, DK, DV, C>;
    constexpr size_t kBytes = L::template bytes<IO>();
    static_assert(kBytes <= 227 * 1024, "shared memory per CTA");
    auto kern = prefill_simt_kernel<MODE, DK, DV, C, IO>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBytes);
    if (err != cudaSuccess) return err;
    timer_begin(a.stream);
    const unsigned grid = (unsigned)(a.cu ? (size_t)a.nseq * a.H : (size_t)a.B * a.H);
    kern<<<grid, kSimtThreads, kBytes, a.stream>>>(
        a.T, a.H, a.cu, static_cast<const IO *>(a.q), static_cast<const IO *>(a.k),
        static_cast<const IO *>(a.v), a.gate, a.beta, a.state, a.z, static_cast<IO *>(a.o),
        a.init_state ? 1 : 0, device_error_word(), a.gate_heads);
    timer_end(a.stream);
    note_launches(1);
    return cudaGetLastError();
}

template <int MODE, int DK, int DV, typename IO>
cudaError_t launch_chunk(const PrefillArgs &a) {
    if (a.chunk == 32) return launch_one<MODE, DK, DV, 32, IO>(a);
    if constexpr (DK == 64 && DV == 64) {
        if (a.chunk == 64) return launch_one<MODE, DK, DV, 64, IO>(a);
    }
    return cudaErrorInvalidValue;
}

template <int MODE, typename IO>
cudaError_t launch_dims(const PrefillArgs &a) {
    if (a.dk == 64 && a.dv == 64) return launch_chunk<MODE, 64, 64, IO>(a);
    if (a.dk == 128 && a.dv == 128) return launch_chunk<MODE, 128, 128, IO>(a);
    if (a.dk == 64 && a.dv == 128) return launch_chunk<MODE, 64, 128, IO>(a);
    if (a.dk == 128 && a.dv == 64) return launch_chunk<MODE, 128, 64, IO>(a);
    return cudaErrorInvalidValue;
}

template <typename IO>
cudaError_t launch_io(const PrefillArgs &a) {
    switch (a.mode) {
        case LA_MODE_ELU1_NORM: return launch_dims<0, IO>(a);
        case LA_MODE_GATED: return launch_dims<1, IO>(a);
        case LA_MODE_GATED_DELTA: return launch_dims<2, IO>(a);
        case LA_MODE_KDA: return launch_dims<3, IO>(a);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

bool prefill_simt_supports(int dtype, int dk, int dv, int chunk, int *resolved) {
    (void)dtype;
    const bool small = (dk == 64 && dv == 64);
    const int c = chunk == 0 ? (small ? 64 : 32) : chunk;
    if (c == 32 || (c == 64 && small)) {
        *resolved = c;
        return true;
    }
    return false;
}

cudaError_t launch_prefill_simt(const PrefillArgs &a) {
    return a.dtype == LA_BF16 ? launch_io<__nv_bfloat16>(a) : launch_io<float>(a);
}

}  // namespace la

// prefill_tc.cu -- chunked prefill on the 5th-generation tensor cores (tcgen05 + TMEM,
// operands staged by TMA), bf16 I/O, d_k = d_v = 128, chunk C = 64, fp32 state.
//
// The method is the chunked form of the lesson page "Linear attention and hybrids",
// section "Three forms of one computation" (inside a chunk the masked C x C matrix,
// across chunks the carried state), with the decay mask of section "Memory must forget:
// decay and gates" and, in mode 2, the Gated DeltaNet update of section "The delta rule
// and Gated DeltaNet".  Per chunk of L <= 64 tokens, with the in-chunk log-gate prefix
// lam_t = sum_{m<=t} log a_m, g_t = exp(lam_t), dec_t = exp(lam_{L-1} - lam_t) (all <= 1):
//
//   G   = [K; Q] K^T                            (rows 0-63: K K^T, rows 64-127: Q K^T)
//   A   = (Q K^T) * exp(lam_t - lam_j), j <= t  (mode 0: phi(Q) phi(K)^T, no decay)
//   modes 0/1:  O  = diag(g) Q S^T + A V          (mode 0: divided by den_t)
//               S <- g_{L-1} S + V^T diag(dec) K
//   mode 2:     Lm = strictly-lower(diag(b) exp(lam_t - lam_j) K K^T),  T = (I + Lm)^-1
//               U^T = V^T (T diag(b))^T,  W^T = K^T (T diag(b g))^T
//               E^T = U^T - S W^T   (the write vectors e_t = b_t (v_t - a_t S_{t-1} k_t))
//               O  = diag(g) Q S^T + A E,   S <- g_{L-1} S + (E^T diag(dec)) K
//
// Products and where they live (M x N x K, tcgen05.mma kind::f16, fp32 accumulators
// in tensor memory):  G 128x64x128, U^T and W^T 128x64x64, Y = S W^T 128x64x128,
// dS = V^T K~ (or E'^T K) 128x128x64, O = Q~ S^T + A V (or A E) 64x128x(128+64).  The
// fp32 state S itself stays in the epilogue threads' registers across chunks (each
// thread owns half a row); each chunk adds dS to it and writes a bf16 copy to shared
// memory as the operand of the next chunk's products.  diag(g) and diag(dec) are folded
// into the operands by scaling the Q and K tiles in shared memory (mode 1) or the E
// tile (mode 2), after K K^T / Q K^T have been formed from the unscaled tiles.
//
// Mode 3 (Kimi Delta Attention, same section: Diag(a_t), one decay per column c of S)
// runs the mode-2 kernel with the decays inside the operands.  With per-channel prefixes
// lam_tc, the pair decay exp(lam_tc - lam_jc) is split between the two factors of the
// product around a reference token, one per token half (15 and 47), so that no factor
// spans more than 16 tokens of decay:
//   G1 = [K~; Q~] Kb^T  (N = 64, kept for rows 32-63),  Kb  = K 2^(lam_47 - lam_j),
//   G0 = [K~; Q~] Kb0^T (N = 32, kept for rows 0-31),   Kb0 = K 2^(lam_15 - lam_j),
//   K~, Q~ = K, Q times 2^(lam_t - lam_ref(t)), in place in the stage;
// then K~ -> K o Gamma (W^T = (K o Gamma)^T (T diag b)^T), Q~ -> Q o Gamma (the O
// product), Kb -> K o 2^(lam_L - lam) (dS = E^T Kb), and S <- S Diag(2^lam_L) + dS.
// Every factor of G stays within 2^120 because G's per-token log2 gates are bounded below
// at -7.5 (a >= 0.0055); the other products take the exact gates (see kda_exact below), and
// the CUDA-core kernel (chunk 32) takes every gate as it is everywhere.
// Kb is written only after the previous chunk's products are done (it is one buffer);
// T diag(b g) is not needed, and its slot holds Kb0; outputs are staged in the chunk's V
// slot, so that Kb takes the output staging slot.
//
// Warp roles (320 threads): warp 0 lane 0 issues TMA loads into a ring of stages;
// warp 1 owns TMEM and lane 0 issues every MMA; warps 2-9 are the epilogue: two warps
// per TMEM lane quarter, each taking one half of the columns.  The schedule per chunk c
// (epilogue: A-epilogue(c), prologue of c+1, state(c), output(c)) lets the tensor core
// form G(c+1) and O(c), dS(c) while the epilogue works on the neighbouring chunk.
// Roles hand off through mbarriers; every wait is bounded (a timeout records an error
// and the CTA winds down: in-flight copies and MMAs are drained before TMEM is freed).
//
// A CTA processes one (batch*head, segment) pair: a contiguous token range of the
// sequence.  With several segments per sequence, three kinds of CTA run:
//   LOCAL       the segment's own state contribution from a zero state (no output),
//   TRANSITION  (modes 2, 3) the segment's state transition matrix, i.e. the same
//               recurrence started from the identity with v = 0 (no output),
//   OUTPUT      the outputs, started from the exact state at the segment start.
// A small combine kernel chains segment starts between the two passes.
#include "la_internal.cuh"
#include "ptx.cuh"
#include "tmap.cuh"
#include "tc_util.cuh"

#include <algorithm>
#include <cfloat>

namespace la {
namespace {

using namespace ptx;
using namespace tc;

constexpr int kC = 64;         // chunk
constexpr int kD = 128;        // d_k = d_v
constexpr int kThreads = 320;  // 10 warps
constexpr int kEpi = 256;      // epilogue threads (warps 2-9)
constexpr uint32_t kTmemCols = 512;
// TMEM column map
constexpr uint32_t kColDS = 0, kColG = 128, kColU = 192, kColW = 256, kColY = 320, kColO = 384;
// Kimi Delta Attention (mode 3): the first-half product G0 (N = 32) borrows the first 32
// U columns, free until the U^T product of the same chunk.
constexpr uint32_t kColG0 = kColU;
// Mode 3 bounds each per-channel log2 gate at -kKdaLog2Clamp (a >= 2^-7.5 = 0.0055) inside
// the Gram products G, so that no operand factor 2^(lambda_t - lambda_ref) over half a
// half-chunk exceeds 2^120; the state-facing operands (K o Gamma, Q o Gamma,
// K o 2^(lambda_L - lambda)) and the state's column decay take the exact gates (kda_exact).
constexpr float kKdaLog2Clamp = 7.5f;

// kLocalTrans (delta rule): one launch of both no-output passes, CTAs [0, split) local,
// [split, 2 split) transition, so that the two share the SMs' waves.
enum Kind { kOutput = 0, kLocal = 1, kTransition = 2, kLocalTrans = 3 };

struct TcParams {
    CUtensorMap tq, tk, tv, to;  // [BH][T][128] bf16, box 64 x 64 (to: output, stores)
    const float *gate;           // [BH][T] or nullptr
    const float *beta;           // [BH][T] (mode 2)
    __nv_bfloat16 *o;            // [BH][T][128]
    // initial state: mode 0 zero, 1 from s_in (+ seg * s_in_seg), 2 identity
    const float *s_in;
    long long s_in_seg;
    int s_in_mode;
    const float *z_in;           // mode 0
    long long z_in_seg;
    // where the final state goes (nullptr: not written); out_last_only: only the last
    // segment writes (OUTPUT kind)
    float *s_out;
    long long s_out_seg;
    float *z_out;
    long long z_out_seg;
    float *gam_out;              // LOCAL, mode 1: product of the segment's gates
    int out_last_only;
    int T, BH, seg_len, nseg;
    unsigned *err;
    // s_in_mode 3 (modes 0/1, outputs pass): the start state of segment `seg` is folded in
    // the kernel from fold_init (nullable: zero) and the local states of the first
    // seg * fold_sub sub-segments, S <- gam_j S + N_j (z <- z + zN_j), instead of being
    // read from a start state that a combine kernel wrote.
    const float *fold_init, *fold_zinit, *fold_loc, *fold_zloc, *fold_gam;
    int fold_sub;
    // Constant per-head gates: gate is [gate_heads], head row bh uses gate[bh % gate_heads]
    // for every token (0: per-token gates [BH][T]).
    int gate_heads;
    // kLocalTrans: CTAs from `split` on run the transition pass and write s_out2
    int split;
    float *s_out2;
    // Packed variable-length sequences (nullptr: dense; nseg = their number).  A CTA of
    // sequence s and head row h takes tokens [cu[s], cu[s+1]) of head row h of the packed
    // [H][T][128] tensors; its state is slot s of the s_in / s_out segment stride.
    const int *cu;
};

// The token range of this CTA: segment `seg` of head row `bh`, or, for packed sequences,
// sequence `seg`.  A cu_seqlens entry outside [0, T] or decreasing is clamped (the CTA
// stays in bounds) and reported in the failure word.
struct CtaRange {
    int bh, seg, tb, te;
};
// Packed sequences are served longest first: the CTAs of the r-th longest sequence (ties by
// index) come r-th in launch order, so that the longest ones start in the first wave instead
// of trailing it.  Every warp ranks the sequences itself (lane s counts the sequences ahead
// of sequence s), so no shared memory or barrier is involved; with more than 128 sequences
// they are taken in order.
__device__ __forceinline__ int packed_sequence_of_rank(const TcParams &p, int r) {
    if (p.nseg > 128) return r;
    auto len = [&](int i) -> int {
        const int a = min(max(p.cu[i], 0), p.T);
        return min(max(p.cu[i + 1], a), p.T) - a;
    };
    const int lane = threadIdx.x & 31;
    int sel = r;
    for (int s0 = 0; s0 < p.nseg; s0 += 32) {
        const int s = s0 + lane;
        bool hit = false;
        if (s < p.nseg) {
            const int ls = len(s);
            int rank = 0;
            for (int j = 0; j < p.nseg; ++j) {
                const int lj = len(j);
                rank += (lj > ls || (lj == ls && j < s)) ? 1 : 0;
            }
            hit = rank == r;
        }
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        if (m) sel = s0 + __ffs(m) - 1;
    }
    return sel;
}
// (RANKED = false: packed sequences in launch order.  Only the outputs passes ever run packed;
// the mode-0 one takes the launch order, its registers having no room for the ranking.)
template <bool RANKED = true>
__device__ __forceinline__ CtaRange cta_range(const TcParams &p, int idx) {
    CtaRange r;
    r.bh = idx % p.BH;
    r.seg = (RANKED && p.cu) ? packed_sequence_of_rank(p, idx / p.BH) : idx / p.BH;
    if (p.cu) {
        const int a = p.cu[r.seg], b = p.cu[r.seg + 1];
        r.tb = min(max(a, 0), p.T);
        r.te = min(max(b, r.tb), p.T);
        if ((a != r.tb || b != r.te) && threadIdx.x == 0 && p.err) atomicOr(p.err, (unsigned)kErrBadInput);
    } else {
        r.tb = r.seg * p.seg_len;
        r.te = min(p.T, r.tb + p.seg_len);
    }
    return r;
}

// Row t of a chunk's output, 32 columns from col, written straight to global memory as
// bf16 (the last, partial chunk of a packed sequence: a 64-row TMA store would write
// into the next sequence's rows).
__device__ __forceinline__ void st_out_row32(const TcParams &p, int bh, int t, int col, const float *v) {
    uint4 *dst = reinterpret_cast<uint4 *>(p.o + ((size_t)bh * p.T + t) * 128 + col);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 w;
        w.x = pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]);
        w.y = pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]);
        w.z = pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]);
        w.w = pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]);
        dst[q] = w;
    }
}

// Start state S[row][c0 .. c0 + 15] of segment `seg` of head bh (modes 0/1).
__device__ __forceinline__ void start_state16(const TcParams &p, int seg, int bh, int row, int c0,
                                              float (&v)[16]) {
    const size_t off = (size_t)bh * 128 * 128 + (size_t)row * 128 + c0;
#pragma unroll
    for (int k = 0; k < 16; ++k) v[k] = 0.f;
    const float *src = nullptr;
    if (p.s_in_mode == 1) src = p.s_in + (size_t)seg * p.s_in_seg + off;
    if (p.s_in_mode == 3) src = p.fold_init ? p.fold_init + off : nullptr;
    if (src) {
#pragma unroll
        for (int k = 0; k < 16; k += 4) {
            const float4 x = *reinterpret_cast<const float4 *>(src + k);
            v[k] = x.x; v[k + 1] = x.y; v[k + 2] = x.z; v[k + 3] = x.w;
        }
    }
    if (p.s_in_mode == 3) {
        const size_t per = (size_t)p.BH * 128 * 128;
        for (int j = 0; j < seg * p.fold_sub; ++j) {
            const float g = p.fold_gam ? p.fold_gam[(size_t)j * p.BH + bh] : 1.f;
            const float *n = p.fold_loc + (size_t)j * per + off;
#pragma unroll
            for (int k = 0; k < 16; k += 4) {
                const float4 x = *reinterpret_cast<const float4 *>(n + k);
                v[k] = fmaf(g, v[k], x.x);
                v[k + 1] = fmaf(g, v[k + 1], x.y);
                v[k + 2] = fmaf(g, v[k + 2], x.z);
                v[k + 3] = fmaf(g, v[k + 3], x.w);
            }
        }
    }
}
// Start value of z[col] of segment `seg` of head bh (mode 0).
__device__ __forceinline__ float start_z(const TcParams &p, int seg, int bh, int col) {
    if (p.s_in_mode == 1) return p.z_in ? p.z_in[(size_t)seg * p.z_in_seg + (size_t)bh * 128 + col] : 0.f;
    if (p.s_in_mode != 3) return 0.f;
    float z = p.fold_zinit ? p.fold_zinit[(size_t)bh * 128 + col] : 0.f;
    for (int j = 0; j < seg * p.fold_sub; ++j) z += p.fold_zloc[((size_t)j * p.BH + bh) * 128 + col];
    return z;
}

struct Small {
    uint64_t full[3], empty[3];
    uint64_t prep_done, g_done, tt_ready, ut_done, w_ready, py_done, e_ready,
        mma2_done, s_ready, fin;
    uint32_t tmem_base;
    int abort;
    int len[2];
    float lam[2][kC];    // in-chunk inclusive prefix of log2(a), per chunk parity
    float bet[2][kC];
    float scan_tmp[2];
};

// Mode 3 (KDA): per-channel decay vectors of a chunk (parity buffer) and the exchange
// between the two token halves of a channel.
struct SmallKda {
    float eref[2][2][128];   // 2^lambda at the two reference tokens (15, 47), per channel
    float edec[2][128];      // 2^(lambda_L - lambda_47): Kb -> K 2^(lambda_L - lambda)
    float egl[2][128];       // 2^lambda_L: the state's column decay over the chunk
    float tot0[128], tot1[128], x15b[128];   // half totals and the second half's prefix at 15
    float tot0u[128], tot1u[128];            // half totals of the unbounded log2 gates
};

// Shared-memory layout (bytes from the 1024-aligned base).
template <int MODE>
struct Lay {
    static constexpr int kStages = MODE >= 2 ? 2 : 3;
    static constexpr uint32_t kStage = 49152;          // [K0][Q0][K1][Q1][V0][V1], 8 KB each
    static constexpr uint32_t kSbf = kStages * kStage; // 32 KB bf16 state, [d_v][d_k]
    static constexpr uint32_t kA = kSbf + 32768;       // 8 KB  A [t][j]
    static constexpr uint32_t kTp = kA + 8192;         // 8 KB  T diag(b)      (mode 2)
    static constexpr uint32_t kTpp = kTp + 8192;       // 8 KB  T diag(b g)    (mode 2)
    static constexpr uint32_t kX = kTpp + 8192;        // 48 KB E | E' | W  or  Lm | Tm | Zs
    static constexpr uint32_t kE = kX, kEp = kX + 16384, kW = kX + 32768;
    static constexpr uint32_t kOst = MODE >= 2 ? kX + 49152 : kA + 8192;   // 16 KB O staging
    static constexpr uint32_t kSmall = kOst + 16384;
    // mode 3: T diag(b g) is not needed (the decay sits in the K operand); its slot holds
    // Kb0 = K 2^(lambda_15 - lambda) (rows 0-31, two 4 KB halves), and the O staging
    // slot holds Kb = K 2^(lambda_47 - lambda) (then K 2^(lambda_L - lambda)); outputs are
    // staged in the chunk's V slot instead.
    static constexpr uint32_t kKb0 = kTpp, kKb = kOst;
    static constexpr uint32_t kKda = (kSmall + sizeof(Small) + 15) & ~15u;
    static constexpr uint32_t kBytes = MODE == 3 ? kKda + sizeof(SmallKda) : kSmall + sizeof(Small);
};
static_assert(Lay<3>::kBytes <= 227 * 1024, "shared memory per CTA");

__device__ __forceinline__ void epi_sync() { named_sync(1, kEpi); }
// Raw gate a_t and beta_t of token `e` of chunk c (64 threads, e < 64), fetched a chunk
// ahead of use so that the global-load latency overlaps the previous chunk's epilogue.
struct GateRaw {
    float a, b;
};
template <int MODE>
__device__ __forceinline__ GateRaw fetch_gates(const TcParams &p, int bh, int tb, int te, int c,
                                               int e) {
    GateRaw r{1.f, 0.f};
    const int t0 = tb + kC * c;
    const int L = min(kC, te - t0);
    if ((MODE == 1 || MODE == 2) && p.gate && e < L)
        r.a = p.gate[p.gate_heads ? (size_t)(bh % p.gate_heads) : (size_t)bh * p.T + t0 + e];
    if (MODE >= 2 && e < L) r.b = p.beta[(size_t)bh * p.T + t0 + e];
    return r;
}

// Gates of chunk c into parity buffer `buf`: log2 prefix and beta (64 threads, e < 64).
template <int MODE>
__device__ __forceinline__ void load_gates(const TcParams &p, Small *sm, int tb, int te, int c,
                                           int buf, int e, GateRaw raw) {
    const int t0 = tb + kC * c;
    const int L = min(kC, te - t0);
    float g = ((MODE == 1 || MODE == 2) && e < L) ? lg2(fmaxf(raw.a, FLT_MIN)) : 0.f;
    const int lane = e & 31;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float n = __shfl_up_sync(0xffffffffu, g, off);
        if (lane >= off) g += n;
    }
    if (lane == 31) sm->scan_tmp[e >> 5] = g;
    named_sync(2, 64);
    if (e >= 32) g += sm->scan_tmp[0];
    sm->lam[buf][e] = g;
    sm->bet[buf][e] = (MODE >= 2 && e < L) ? raw.b : 0.f;
    if (e == 0) sm->len[buf] = L;
    named_sync(2, 64);
    (void)p;
}

// phi(x) = elu(x) + 1 = max(x, 0) + exp(min(x, 0)) on a packed pair of bf16, in bf16x2
// arithmetic (the inputs and results are bf16 MMA operands).
__device__ __forceinline__ uint32_t phi_bf16x2(uint32_t x) {
    uint32_t r;
    asm("{\n\t.reg .b32 lo, hi, ex;\n\t"
        "min.bf16x2 lo, %1, %2;\n\t"
        "max.bf16x2 hi, %1, %2;\n\t"
        "mul.rn.bf16x2 lo, lo, %3;\n\t"
        "ex2.approx.ftz.bf16x2 ex, lo;\n\t"
        "add.rn.bf16x2 %0, hi, ex;\n\t}"
        : "=r"(r)
        : "r"(x), "r"(0u), "r"(0x3FB93FB9u));   // bf16x2 of log2(e) = 1.4453 (0x3FB9)
    return r;
}


template <int MODE, int KIND>
__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(const __grid_constant__ TcParams p) {
    static_assert(MODE == 2 || MODE == 3, "this kernel serves the delta rule (modes 2, 3)");
    constexpr bool kKda = (MODE == 3);   // per-channel decay: it sits in the K / Q operands
    using Y = Lay<MODE>;
    constexpr int NST = Y::kStages;
    constexpr bool kOut = (KIND == kOutput);
    // transition CTAs: the recurrence from the identity with v = 0 (no V, no outputs)
    const bool trans = (KIND == kTransition) || (KIND == kLocalTrans && (int)blockIdx.x >= p.split);
    const bool needV = !trans;

    // 128B-swizzled operand tiles need 1024-byte aligned atoms.  The buffer is declared
    // with that alignment and never re-aligned by integer arithmetic: pointers derived
    // from it keep the shared address space.
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sb = smem_u32(smem_raw);
    if (sb & 1023u) {
        if (threadIdx.x == 0 && p.err) atomicOr(p.err, (unsigned)kErrBadLaunch);
        return;
    }
    Small *sm = reinterpret_cast<Small *>(smem_raw + Y::kSmall);
    SmallKda *sk = reinterpret_cast<SmallKda *>(smem_raw + (kKda ? Y::kKda : Y::kSmall));   // mode 3

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const CtaRange rng = cta_range<KIND == kOutput>(p, (int)blockIdx.x - (KIND == kLocalTrans && trans ? p.split : 0));
    const int bh = rng.bh, seg = rng.seg, tb = rng.tb, te = rng.te;
    if (te <= tb) return;   // an empty packed sequence: nothing to read or write
    const int nch = (te - tb + kC - 1) / kC;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&sm->full[s], 1);
            mbar_init(&sm->empty[s], 1);
        }
        mbar_init(&sm->prep_done, 1);
        mbar_init(&sm->g_done, 1);
        mbar_init(&sm->tt_ready, 1);
        mbar_init(&sm->ut_done, 1);
        mbar_init(&sm->w_ready, 1);
        mbar_init(&sm->py_done, 1);
        mbar_init(&sm->e_ready, 1);
        mbar_init(&sm->mma2_done, 1);
        mbar_init(&sm->s_ready, 1);
        mbar_init(&sm->fin, 1);
        sm->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = sm->tmem_base;
    volatile int *abort = &sm->abort;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&p.tk);
            if (kOut) tma_prefetch_desc(&p.tq);
            if (needV) tma_prefetch_desc(&p.tv);
            int issued[NST];
            for (int s = 0; s < NST; ++s) issued[s] = 0;
            for (int c = 0; c < nch; ++c) {
                const int s = c % NST, u = c / NST;
                if (u >= 1 && !mbar_wait(&sm->empty[s], (u - 1) & 1, abort, p.err)) break;
                const uint32_t st = sb + s * Y::kStage;
                const int t = tb + kC * c;
                const uint32_t bytes = 16384u * (1u + (kOut ? 1u : 0u) + (needV ? 1u : 0u));
                mbar_arrive_expect_tx(&sm->full[s], bytes);
                tma_load_3d(st + 0, &p.tk, 0, t, bh, &sm->full[s]);
                tma_load_3d(st + 16384, &p.tk, 64, t, bh, &sm->full[s]);
                if (kOut) {
                    tma_load_3d(st + 8192, &p.tq, 0, t, bh, &sm->full[s]);
                    tma_load_3d(st + 24576, &p.tq, 64, t, bh, &sm->full[s]);
                }
                if (needV) {
                    tma_load_3d(st + 32768, &p.tv, 0, t, bh, &sm->full[s]);
                    tma_load_3d(st + 40960, &p.tv, 64, t, bh, &sm->full[s]);
                }
                issued[s] = u + 1;
            }
            // no copy may still be writing shared memory when the CTA exits
            for (int s = 0; s < NST; ++s)
                if (issued[s] > 0) drain_wait(&sm->full[s], (issued[s] - 1) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t sbf = sb + Y::kSbf, at = sb + Y::kA, tp = sb + Y::kTp,
                           tpp = sb + Y::kTpp, et = sb + Y::kE, ept = sb + Y::kEp,
                           wt = sb + Y::kW;
            const uint32_t id_g = idesc_bf16(128, 64, false, false);
            const uint32_t id_g0 = idesc_bf16(128, 32, false, false);   // mode 3
            const uint32_t kb = sb + Y::kKb, kb0 = sb + Y::kKb0;           // mode 3
            const uint32_t id_uw = idesc_bf16(128, 64, true, false);
            const uint32_t id_y = idesc_bf16(128, 64, false, true);
            const uint32_t id_o1 = idesc_bf16(64, 128, false, false);
            const uint32_t id_o2 = idesc_bf16(64, 128, false, MODE < 2);
            const uint32_t id_ds = idesc_bf16(128, 128, MODE < 2, true);
            for (int c = 0; c < nch; ++c) {
                const int s = c % NST, u = c / NST;
                const uint32_t par = c & 1;
                const uint32_t st = sb + s * Y::kStage;
                if (!mbar_wait(&sm->full[s], u & 1, abort, p.err)) break;
                if (!mbar_wait(&sm->prep_done, par, abort, p.err)) break;
                tc_fence_after();
                if constexpr (kKda) {
                    // G1 = [K~; Q~] Kb^T (N=64, rows of the second token half) and
                    // G0 = [K~; Q~] Kb0^T (N=32, rows of the first half); the operands carry
                    // the per-channel decays relative to tokens 47 and 15
                    mma_chain<8, true, true, 16384, 8192>(tm + kColG, dk(st), dk(kb), id_g, false);
                    mma_chain<8, true, true, 16384, 4096>(tm + kColG0, dk(st), dk(kb0), id_g0, false);
                    mma_commit(&sm->g_done);
                } else {
                    // G = [K; Q] K^T   (M=128, N=64, K=128)
                    mma_chain<8, true, true>(tm + kColG, dk(st), dk(st), id_g, false);
                    mma_commit(&sm->g_done);
                }
                {
                    if (!mbar_wait(&sm->tt_ready, par, abort, p.err)) break;
                    tc_fence_after();
                    if (needV)   // U^T = V^T (T diag b)^T
                        mma_chain<4, false, true>(tm + kColU, dmn(st + 32768, 8192), dk(tp), id_uw, false);
                    // W^T = K^T (T diag(b g))^T; mode 3: (K o Gamma)^T (T diag b)^T
                    mma_chain<4, false, true>(tm + kColW, dmn(st, 16384), dk(kKda ? tp : tpp), id_uw, false);
                    mma_commit(&sm->ut_done);
                    if (!mbar_wait(&sm->w_ready, par, abort, p.err)) break;
                    if (!mbar_wait(&sm->s_ready, par, abort, p.err)) break;
                    tc_fence_after();
                    // Y = S W^T
                    mma_chain<8, true, false>(tm + kColY, dk(sbf), dmn(wt, 8192), id_y, false);
                    mma_commit(&sm->py_done);
                    if (!mbar_wait(&sm->e_ready, par, abort, p.err)) break;
                    tc_fence_after();
                }
                if (kOut) {
                    // O = Q~ S^T + A E   (M=64, N=128; Q~ = diag(g) Q was scaled in place)
                    mma_chain<8, true, true>(tm + kColO, dk(st + 8192), dk(sbf), id_o1, false);
                    mma_chain<4, true, true>(tm + kColO, dk(at), dk(et), id_o2, true);
                }
                // dS = (E^T diag dec) K   (M=128, N=128); mode 3: E^T (K o 2^(lambda_L - lambda))
                if constexpr (kKda)
                    mma_chain<4, true, false>(tm + kColDS, dk(et), dmn(kb, 8192), id_ds, false);
                else
                    mma_chain<4, true, false>(tm + kColDS, dk(ept), dmn(st, 16384), id_ds, false);
                mma_commit(&sm->mma2_done);
            }
            // nothing may still write TMEM when it is freed
            mma_commit(&sm->fin);
            drain_wait(&sm->fin, 0);
        }
    } else {
        // ------------------------------------------------------------ epilogue warps 2-9
        const int e = threadIdx.x - 64;            // 0..255
        const int q = warp & 3;                    // TMEM lane quarter of this warp
        const int h = (warp - 2) >> 2;             // column half
        const int row = 32 * q + lane;             // TMEM lane = tile row
        const uint32_t tl = tm + ((uint32_t)(32 * q) << 16);
        const uint32_t sbf = sb + Y::kSbf;
        float *Lm = reinterpret_cast<float *>(smem_raw + Y::kX);
        float *Tm = Lm + 64 * kLmStride;
        float *Zs = Tm + 64 * kLmStride;

        // ---- initial state: this thread's half row of S in registers, bf16 copy in smem
        float Sr[64];
        {
            const float *src = nullptr;
            const int s_in_mode = trans ? 2 : p.s_in_mode;
            if (s_in_mode == 1)
                src = p.s_in + (size_t)seg * p.s_in_seg + (size_t)bh * kD * kD + (size_t)row * kD;
#pragma unroll
            for (int j = 0; j < 64; ++j) {
                const int col = 64 * h + j;
                Sr[j] = src ? src[col] : ((s_in_mode == 2 && col == row) ? 1.f : 0.f);
            }
#pragma unroll
            for (int g = 0; g < 4; ++g) st_row_bf16x16(sbf + h * 16384, row, 2 * g, Sr + 16 * g);
            fence_async_smem();
            epi_sync();
            if (e == 0) mbar_arrive(&sm->s_ready);
        }

        // ---- mode 3: thread e owns channel kch for the token half khh of every chunk
        const int kch = e & 127, khh = e >> 7;
        float kx[32];            // inclusive prefix of the bounded log2 gates within the half
        float kx15 = 0.f;        // the prefix at the half's reference token (15 or 47)
        float kref = 0.f;        // exponent base of Kb: lambda_47 in this thread's prefix units
        bool kcl = false;        // some log2 gate of the chunk was below -kKdaLog2Clamp
        // L2 prefetch of chunk c's gate rows (64 tokens x 512 B: one line per thread)
        auto kda_prefetch = [&](int c) {
            const int t0 = tb + kC * c, tok = e >> 2;
            if (p.gate && tok < min(kC, te - t0))
                prefetch_l2(p.gate + ((size_t)bh * p.T + t0 + tok) * kD + 32 * (e & 3));
        };
        auto kda_load = [&](int c, float (&g)[32]) {
            const int t0 = tb + kC * c;
            const int L = min(kC, te - t0);
            const float *gp = p.gate + ((size_t)bh * p.T + t0 + 32 * khh) * kD + kch;
#pragma unroll
            for (int i = 0; i < 32; ++i) g[i] = (p.gate && 32 * khh + i < L) ? gp[(size_t)i * kD] : 1.f;
        };
        // prefixes, the exchange between the halves, and the chunk's decay vectors
        auto kda_prefix = [&](int c, const float (&g)[32]) {
            float acc = 0.f;
            bool low = false;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float l = lg2(fmaxf(g[i], FLT_MIN));
                low |= l < -kKdaLog2Clamp;
                acc += fmaxf(l, -kKdaLog2Clamp);
                kx[i] = acc;
            }
            kx15 = kx[15];
            if (khh == 0) {
                sk->tot0[kch] = acc;
            } else {
                sk->tot1[kch] = acc;
                sk->x15b[kch] = kx15;
            }
            kcl = named_sync_any(1, kEpi, low);   // (the epilogue barrier, with an OR)
            const float tot0 = sk->tot0[kch];
            kref = (khh == 0) ? tot0 + sk->x15b[kch] : kx15;
            if (khh == 0) {
                const int b2 = c & 1;
                const float lL = tot0 + sk->tot1[kch];
                sk->eref[b2][0][kch] = ex2(kx15);
                sk->eref[b2][1][kch] = ex2(kref);
                sk->edec[b2][kch] = ex2(lL - kref);
                sk->egl[b2][kch] = ex2(lL);
            }
        };
        // chunk c's operands: K~ = K 2^(lambda - lambda_ref), Q~ likewise (in place; the
        // reference is token 15 for the first half, 47 for the second), Kb and Kb0.  Runs
        // once the previous chunk's products are done (Kb is a single buffer); then G may go.
        auto kda_scale = [&](int c) {
            const uint32_t st = (c % NST) * Y::kStage;
            const uint32_t cb = (uint32_t)(kch >> 6), cc = (uint32_t)(kch & 63);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const uint32_t t = 32 * khh + i;
                const uint32_t o = sw128_off(t, cc >> 3) + ((cc & 7) << 1);
                __nv_bfloat16 *kp = reinterpret_cast<__nv_bfloat16 *>(smem_raw + st + cb * 16384 + o);
                const float kv = __bfloat162float(*kp);
                const float fa = ex2(kx[i] - kx15);
                *kp = __float2bfloat16_rn(kv * fa);
                if (kOut) {
                    __nv_bfloat16 *qp = kp + 4096;   // the Q tile sits 8 KB after the K tile
                    *qp = __float2bfloat16_rn(__bfloat162float(*qp) * fa);
                }
                *reinterpret_cast<__nv_bfloat16 *>(smem_raw + Y::kKb + cb * 8192 + o) =
                    __float2bfloat16_rn(kv * ex2(kref - kx[i]));
                if (khh == 0)
                    *reinterpret_cast<__nv_bfloat16 *>(smem_raw + Y::kKb0 + cb * 4096 + o) =
                        __float2bfloat16_rn(kv * ex2(kx15 - kx[i]));
            }
            fence_async_smem();
            epi_sync();
            if (e == 0) mbar_arrive(&sm->prep_done);
        };
        // Chunk c's state-facing operands with the exact gates, in a chunk where some log2
        // gate is below -kKdaLog2Clamp (kcl): the Gram products G keep the bounded gates
        // (their factors around the reference tokens must stay finite), while K o Gamma,
        // Q o Gamma, K o 2^(lambda_L - lambda) and the state's column decay 2^lambda_L need
        // no reference and take every gate as it is.  Each thread rescales its own channel
        // and token half by 2^(lambda_exact - lambda_bounded) <= 1 (and the corresponding
        // ratio for Kb), after the per-channel conversion of the A-epilogue.
        auto kda_exact = [&](int c, int b2) {
            const int t0 = tb + kC * c;
            const int L = min(kC, te - t0);
            const float *gp = p.gate + ((size_t)bh * p.T + t0 + 32 * khh) * kD + kch;
            float accu = 0.f;
            for (int i = 0; i < 32; ++i)
                accu += (p.gate && 32 * khh + i < L) ? lg2(fmaxf(gp[(size_t)i * kD], FLT_MIN)) : 0.f;
            if (khh == 0) sk->tot0u[kch] = accu;
            else sk->tot1u[kch] = accu;
            epi_sync();
            const float tot0 = sk->tot0[kch], tot0u = sk->tot0u[kch];
            const float lL = tot0 + sk->tot1[kch], lLu = tot0u + sk->tot1u[kch];
            const float base = khh ? tot0 : 0.f, baseu = khh ? tot0u : 0.f;
            const uint32_t stg = (c % NST) * Y::kStage;
            const uint32_t cb = (uint32_t)(kch >> 6), cc = (uint32_t)(kch & 63);
            float x = 0.f, xu = 0.f;
            for (int i = 0; i < 32; ++i) {
                const float l = (p.gate && 32 * khh + i < L) ? lg2(fmaxf(gp[(size_t)i * kD], FLT_MIN)) : 0.f;
                x += fmaxf(l, -kKdaLog2Clamp);
                xu += l;
                const float lam_b = base + x, lam_u = baseu + xu;
                const float fk = ex2(lam_u - lam_b);                  // K o Gamma, Q o Gamma
                const float fb = ex2((lLu - lam_u) - (lL - lam_b));   // K o 2^(lambda_L - lambda)
                if (fk == 1.f && fb == 1.f) continue;
                const uint32_t tt = 32 * khh + i;
                const uint32_t o = sw128_off(tt, cc >> 3) + ((cc & 7) << 1);
                __nv_bfloat16 *kp = reinterpret_cast<__nv_bfloat16 *>(smem_raw + stg + cb * 16384 + o);
                *kp = __float2bfloat16_rn(__bfloat162float(*kp) * fk);
                if (kOut) {
                    __nv_bfloat16 *qp = kp + 4096;
                    *qp = __float2bfloat16_rn(__bfloat162float(*qp) * fk);
                }
                __nv_bfloat16 *bp = reinterpret_cast<__nv_bfloat16 *>(smem_raw + Y::kKb + cb * 8192 + o);
                *bp = __float2bfloat16_rn(__bfloat162float(*bp) * fb);
            }
            if (khh == 0) sk->egl[b2][kch] = ex2(lLu);
        };
        (void)kda_prefetch; (void)kda_load; (void)kda_prefix; (void)kda_scale; (void)kda_exact;

        // ---- chunk prologue: gates; releases G's inputs to the MMA (mode 3: kda_scale does)
        auto prep = [&](int c, GateRaw raw) -> bool {
            const int s = c % NST, u = c / NST;
            float kg[32];
            if constexpr (kKda) kda_load(c, kg);
            if (e < 64) load_gates<MODE>(p, sm, tb, te, c, c & 1, e, raw);
            mbar_wait(&sm->full[s], u & 1, abort, p.err);
            epi_sync();
            if (*abort) return false;
            if constexpr (kKda) kda_prefix(c, kg);
            epi_sync();
            if (!kKda && e == 0) mbar_arrive(&sm->prep_done);
            return true;
        };

        bool ok = prep(0, e < 64 ? fetch_gates<MODE>(p, bh, tb, te, 0, e) : GateRaw{1.f, 0.f});
        if constexpr (kKda) {
            if (ok) kda_scale(0);
        }
        for (int c = 0; c < nch && ok; ++c) {
            const int s = c % NST, buf = c & 1;
            const uint32_t par = c & 1;
            const uint32_t st = sb + s * Y::kStage;
            const int t0 = tb + kC * c;
            const int L = sm->len[buf];
            const float *lam = sm->lam[buf];
            const float lamL = lam[kC - 1];
            // gates of the next chunk: issue the global loads now, use them in its prologue
            GateRaw next_raw{1.f, 0.f};
            if (c + 1 < nch && e < 64) next_raw = fetch_gates<MODE>(p, bh, tb, te, c + 1, e);
            if (kKda && c + 1 < nch) kda_prefetch(c + 1);

            // ---- A-epilogue: masks and decays of G; operand scaling
            mbar_wait(&sm->g_done, par, abort, p.err);
            epi_sync();
            if (*abort) break;
            tc_fence_after();
            if (kKda && kOut && c >= 1 && e == 0) {
                // chunk c-1's outputs were staged in its V slot: release that stage once
                // the TMA store has read them
                tma_store_wait_read<0>();
                mbar_arrive(&sm->empty[(c - 1) % NST]);
            }
            if constexpr (kKda) {
                // G1 holds the rows of the second token half, G0 (32 columns) those of the
                // first; entries above the diagonal may be huge or not finite and are dropped
                const bool second = (q & 1) != 0;
                float v[32];
                if (second) {
                    tmem_ld32(tl + kColG + 32 * h, v);
                } else if (h == 0) {
                    tmem_ld32(tl + kColG0, v);
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = 0.f;
                }
                if (q >= 2 && kOut) {
                    const int i = row - 64;
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = (32 * h + j <= i) ? v[j] : 0.f;
                    st_row_bf16x16(sb + Y::kA, i, 4 * h, v);
                    st_row_bf16x16(sb + Y::kA, i, 4 * h + 2, v + 16);
                } else if (q < 2) {
                    const int r = row;
                    const float br = sm->bet[buf][r];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int jj = 32 * h + j;
                        Lm[r * kLmStride + jj] = (jj < r) ? br * v[j] : 0.f;
                    }
                }
            } else if (q >= 2 && kOut) {
                // rows i of Q K^T -> A tile, columns j in [32h, 32h + 32)
                const int i = row - 64;
                float v[32];
                tmem_ld32(tl + kColG + 32 * h, v);
                const float li = lam[i];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int jj = 32 * h + j;
                    v[j] = (jj <= i) ? v[j] * ex2(li - lam[jj]) : 0.f;
                }
                st_row_bf16x16(sb + Y::kA, i, 4 * h, v);
                st_row_bf16x16(sb + Y::kA, i, 4 * h + 2, v + 16);
            } else if (q < 2) {
                // rows r of K K^T -> Lm (strictly lower), columns j in [32h, 32h + 32)
                const int r = row;
                const float br = sm->bet[buf][r], lr = lam[r];
                float v[32];
                tmem_ld32(tl + kColG + 32 * h, v);
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int jj = 32 * h + j;
                    Lm[r * kLmStride + jj] = (jj < r) ? br * ex2(lr - lam[jj]) * v[j] : 0.f;
                }
            }
            if constexpr (kKda) {
                // after G: K~ -> K o Gamma (the W^T operand), Q~ -> Q o Gamma (the O
                // operand), Kb -> K o 2^(lambda_L - lambda) (the dS operand), in place;
                // Gamma = 2^lambda, every factor <= 1
                const float *ed = sk->edec[buf];
#pragma unroll
                for (int it = 0; it < 4; ++it) {
                    const int n = e + kEpi * it;   // 16-byte chunk of a 64 x 128 tile
                    const int half = n >> 9, rr = (n & 511) >> 3, pc = n & 7;
                    const int c0 = 64 * half + 8 * (pc ^ (rr & 7));
                    const float *f = sk->eref[buf][rr >= 32 ? 1 : 0];
                    const float4 f0 = *reinterpret_cast<const float4 *>(f + c0);
                    const float4 f1 = *reinterpret_cast<const float4 *>(f + c0 + 4);
                    const uint32_t ka = st + half * 16384 + (n & 511) * 16;
                    sts128(ka, scale_bf16x8v(lds128(ka), f0, f1));
                    if (kOut) sts128(ka + 8192, scale_bf16x8v(lds128(ka + 8192), f0, f1));
                    const float4 d0 = *reinterpret_cast<const float4 *>(ed + c0);
                    const float4 d1 = *reinterpret_cast<const float4 *>(ed + c0 + 4);
                    const uint32_t ba = sb + Y::kKb + half * 8192 + (n & 511) * 16;
                    sts128(ba, scale_bf16x8v(lds128(ba), d0, d1));
                }
                if (kcl) {   // uniform over the epilogue threads
                    epi_sync();
                    kda_exact(c, buf);
                }
            } else if (kOut) {
                // after G: Q <- diag(g) Q in place
                uint4 wq[4];
#pragma unroll
                for (int it = 0; it < 4; ++it) {
                    const int n = e + kEpi * it;
                    wq[it] = lds128(st + 8192 + (n >> 9) * 16384 + (n & 511) * 16);
                }
#pragma unroll
                for (int it = 0; it < 4; ++it) {
                    const int n = e + kEpi * it;
                    sts128(st + 8192 + (n >> 9) * 16384 + (n & 511) * 16,
                           scale_bf16x8(wq[it], ex2(lam[(n & 511) >> 3])));
                }
            }
            fence_async_smem();
            tc_fence_before();
            epi_sync();

            {
                // ---- T = (I + Lm)^-1;  T diag(b), T diag(b g) as bf16 MMA operands
                invert_unit_lower<1, kEpi>(Lm, Tm, Zs, e);
                if (e < 128) {
                    const int t = e >> 1, hh = e & 1;
                    for (int g = 0; g < 2; ++g) {
                        const int j0 = 32 * hh + 16 * g;
                        float v1[16], v2[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float tv = Tm[t * kLmStride + j0 + j] * sm->bet[buf][j0 + j];
                            v1[j] = tv;
                            v2[j] = kKda ? 0.f : tv * ex2(lam[j0 + j]);
                        }
                        st_row_bf16x16(sb + Y::kTp, t, j0 >> 3, v1);
                        // mode 3 keeps Kb0 in this slot: its W^T uses T diag(b)
                        if (!kKda) st_row_bf16x16(sb + Y::kTpp, t, j0 >> 3, v2);
                    }
                }
                fence_async_smem();
                epi_sync();
                if (e == 0) mbar_arrive(&sm->tt_ready);
                // ---- W^T (row = d_k index) -> bf16 tile [d_k][t] (MN-major B of S W^T)
                mbar_wait(&sm->ut_done, par, abort, p.err);
                epi_sync();
                if (*abort) break;
                tc_fence_after();
                {
                    float v[32];
                    tmem_ld32(tl + kColW + 32 * h, v);
                    st_row_bf16x16(sb + Y::kW, row, 4 * h, v);
                    st_row_bf16x16(sb + Y::kW, row, 4 * h + 2, v + 16);
                }
                fence_async_smem();
                tc_fence_before();
                epi_sync();
                if (e == 0) mbar_arrive(&sm->w_ready);
                // ---- E^T = U^T - S W^T (row = d_v index); E^T diag(dec)
                mbar_wait(&sm->py_done, par, abort, p.err);
                epi_sync();
                if (*abort) break;
                tc_fence_after();
                {
                    float y[32], uu[32], ev[32];
                    tmem_ld32(tl + kColY + 32 * h, y);
                    if (needV) tmem_ld32(tl + kColU + 32 * h, uu);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int t = 32 * h + j;
                        const float ex = (t < L) ? ((needV ? uu[j] : 0.f) - y[j]) : 0.f;
                        y[j] = ex;
                        ev[j] = (!kKda && t < L) ? ex * ex2(lamL - lam[t]) : 0.f;
                    }
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
                        st_row_bf16x16(sb + Y::kE, row, 4 * h + 2 * g, y + 16 * g);
                        // mode 3 takes the decay in the K operand of dS (Kb): no E'
                        if (!kKda) st_row_bf16x16(sb + Y::kEp, row, 4 * h + 2 * g, ev + 16 * g);
                    }
                }
                fence_async_smem();
                tc_fence_before();
                epi_sync();
                if (e == 0) mbar_arrive(&sm->e_ready);
            }

            // ---- prologue of the next chunk overlaps the products of this one
            if (c + 1 < nch && !prep(c + 1, next_raw)) break;

            // ---- state: S <- g_{L-1} S + dS in registers; bf16 copy for the next chunk
            mbar_wait(&sm->mma2_done, par, abort, p.err);
            if (kOut && e == 0) tma_store_wait_read<0>();   // O staging free again
            epi_sync();
            if (*abort) break;
            tc_fence_after();
            const bool last = (c + 1 == nch);
            // mode 3: the next chunk's operands now that this chunk's products are done;
            // G(c+1) runs while this chunk's state and outputs are finished
            if (kKda && !last) kda_scale(c + 1);
            {
                const float gC = ex2(lamL);
                {
                    float v[64];
                    tmem_ld64(tl + kColDS + 64 * h, v);
                    if constexpr (kKda) {   // S <- S Diag(2^lambda_L) + dS: one decay per column
                        const float *gl = sk->egl[buf] + 64 * h;
#pragma unroll
                        for (int j = 0; j < 64; ++j) Sr[j] = fmaf(gl[j], Sr[j], v[j]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 64; ++j) Sr[j] = fmaf(gC, Sr[j], v[j]);
                    }
                }
                if (!last) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) st_row_bf16x16(sbf + h * 16384, row, 2 * g, Sr + 16 * g);
                }
                if (last) {
                    float *out = (KIND == kLocalTrans && trans) ? p.s_out2 : p.s_out;
                    const bool write = out && (!p.out_last_only || seg == p.nseg - 1);
                    if (write) {
                        float *dst = out + (size_t)seg * p.s_out_seg + (size_t)bh * kD * kD +
                                     (size_t)row * kD + 64 * h;
#pragma unroll
                        for (int j = 0; j < 64; j += 4)
                            *reinterpret_cast<float4 *>(dst + j) =
                                make_float4(Sr[j], Sr[j + 1], Sr[j + 2], Sr[j + 3]);
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            epi_sync();
            if (e == 0) {
                mbar_arrive(&sm->s_ready);
                // mode 3 stages the outputs in this stage's V slot: released after the store
                if (!(kKda && kOut)) mbar_arrive(&sm->empty[s]);
            }

            // ---- outputs: row t of O (M=64 layout: lane (t % 16) + 32 (t / 16)), half h,
            // staged as bf16 in shared memory and written by two TMA stores (rows past the
            // end of the sequence are clipped by the tensor map)
            if (kOut) {
                const int t = 16 * q + lane;
                const bool has = lane < 16 && t < L;
                const bool direct = p.cu && L < kC;   // partial chunk of a packed sequence
                // mode 3: the V slot of this chunk's stage (V is dead after U^T)
                const uint32_t obase = kKda ? st + 32768 : sb + Y::kOst;
                const uint32_t ost = obase + h * 8192;
#pragma unroll
                for (int sub = 0; sub < 2; ++sub) {
                    float v[32];
                    tmem_ld32(tl + kColO + 64 * h + 32 * sub, v);
                    if (has && direct) {
                        st_out_row32(p, bh, t0 + t, 64 * h + 32 * sub, v);
                    } else if (has) {
                        st_row_bf16x16(ost, t, 4 * sub, v);
                        st_row_bf16x16(ost, t, 4 * sub + 2, v + 16);
                    }
                }
                fence_async_smem();
                tc_fence_before();
                epi_sync();
                if (e == 0 && !direct) {
                    tma_store_3d(&p.to, obase, 0, t0, bh);
                    tma_store_3d(&p.to, obase + 8192, 64, t0, bh);
                    tma_store_commit();
                }
            }
        }
    }
    if (kOut && warp >= 2 && threadIdx.x == 64) tma_store_wait_all<0>();   // outputs landed
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tm, kTmemCols);
    }
}

// ------------------------------------------------------------------ modes 0 / 1
// The two modes without the delta-rule solve run a dedicated kernel of 12 warps:
//   warp 0      TMA producer (a ring of three stages of K, Q, V tiles),
//   warp 1      owns TMEM; lane 0 issues every MMA,
//   warps 2-9   epilogue: A tile, outputs, and the fp32 state (in registers),
//   warps 10-11 chunk preparation, running ahead of the epilogue: the in-chunk gate
//               prefix (mode 1), the feature map phi = elu + 1 applied in place to the
//               Q and K tiles, the running normaliser z and phi(q_t).z (mode 0), and,
//               in the LOCAL pass, the decayed K~ = diag(dec) K (mode 1).
// Per chunk c of the OUTPUT pass the tensor core forms G(c+1) = Q K^T (M=64) while the
// epilogue is still on chunk c, then Q S^T, A V (M=64) and dS = V^T K~ (M=128) of chunk c.
// The epilogue turns G(c+1) into the A tile of chunk c+1 while those products run,
// then writes the outputs of chunk c and adds dS to its register-resident state.  The
// LOCAL pass (no outputs) double-buffers dS so that the state update of chunk c
// overlaps the product of chunk c+1.
//
// Every hand-off is an mbarrier whose next phase cannot complete before its waiter has
// consumed the current one: a stage is released only when both the tensor core (commit)
// and the epilogue (after its last use of the chunk) are done with it, and the
// per-chunk barriers that can run ahead are double-buffered by chunk parity.  One
// thread per role polls each barrier, with a bound; the others meet it at a named
// barrier that also ORs the abandon decision, so that every thread leaves together.
constexpr int kThreads01 = 384;                 // 12 warps
constexpr uint32_t kColG01 = 128;               // two 64-column G buffers (M=64)
constexpr uint32_t kColO01 = 256, kColP01 = 384;

struct Small01 {
    uint64_t full[3], empty[3], prep_done[3];
    uint64_t g_done[2], a_ready[2], ds_done[2], ds_free[2];
    uint64_t s_ready, mma2_done, fin;
    uint32_t tmem_base;
    int abort;
    int len[8];
    float lam[8][kC];       // in-chunk inclusive prefix of log2(a), chunk mod 8
    float scan_tmp[2];
};
struct Lay01 {
    static constexpr int kStages = 3;
    static constexpr uint32_t kStage = 49152;             // [K0][Q0][K1][Q1][V0][V1], 8 KB each
    static constexpr uint32_t kSbf = kStages * kStage;    // 32 KB bf16 state [d_v][d_k]
    static constexpr uint32_t kA = kSbf + 32768;          // 2 x 8 KB A tiles [t][j]
    static constexpr uint32_t kOst = kA + 16384;          // 16 KB output staging
    static constexpr uint32_t kSmall = kOst + 16384;
    static constexpr uint32_t kBytes = kSmall + sizeof(Small01);
};
static_assert(Lay01::kBytes <= 227 * 1024, "shared memory per CTA");

__device__ __forceinline__ float ld_gate(const TcParams &p, int bh, int t0, int L, int i) {
    float a = 1.f;
    const size_t off = p.gate_heads ? (size_t)(bh % p.gate_heads) : (size_t)bh * p.T + t0 + i;
    if (i < L) asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(a) : "l"(p.gate + off));
    return a;
}

template <int MODE, int KIND>
__global__ void __launch_bounds__(kThreads01, 1) prefill01_kernel(const __grid_constant__ TcParams p) {
    using Y = Lay01;
    constexpr int NST = Y::kStages;
    constexpr bool kOut = (KIND == kOutput);
    static_assert(MODE == 1, "this kernel serves the scalar-gated mode");
    static_assert(KIND == kOutput || KIND == kLocal, "no transition pass without the delta rule");

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sb = smem_u32(smem_raw);
    if (sb & 1023u) {
        if (threadIdx.x == 0 && p.err) atomicOr(p.err, (unsigned)kErrBadLaunch);
        return;
    }
    Small01 *sm = reinterpret_cast<Small01 *>(smem_raw + Y::kSmall);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const CtaRange rng = cta_range<KIND == kOutput>(p, (int)blockIdx.x);
    const int bh = rng.bh, seg = rng.seg, tb = rng.tb, te = rng.te;
    if (te <= tb) return;   // an empty packed sequence: nothing to read or write
    const int nch = (te - tb + kC - 1) / kC;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&sm->full[s], 1);
            mbar_init(&sm->empty[s], 2);     // tensor-core commit + epilogue
            mbar_init(&sm->prep_done[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm->g_done[b], 1);
            mbar_init(&sm->a_ready[b], 1);
            mbar_init(&sm->ds_done[b], 1);
            mbar_init(&sm->ds_free[b], 1);
        }
        mbar_init(&sm->s_ready, 1);
        mbar_init(&sm->mma2_done, 1);
        mbar_init(&sm->fin, 1);
        sm->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = sm->tmem_base;
    volatile int *abort = &sm->abort;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&p.tk);
            tma_prefetch_desc(&p.tv);
            if (kOut) tma_prefetch_desc(&p.tq);
            int issued[NST];
            for (int s = 0; s < NST; ++s) issued[s] = 0;
            for (int c = 0; c < nch; ++c) {
                const int s = c % NST, u = c / NST;
                if (u >= 1 && !mbar_wait(&sm->empty[s], (u - 1) & 1, abort, p.err)) break;
                const uint32_t st = sb + s * Y::kStage;
                const int t = tb + kC * c;
                mbar_arrive_expect_tx(&sm->full[s], kOut ? 49152u : 32768u);
                tma_load_3d(st + 0, &p.tk, 0, t, bh, &sm->full[s]);
                tma_load_3d(st + 16384, &p.tk, 64, t, bh, &sm->full[s]);
                if (kOut) {
                    tma_load_3d(st + 8192, &p.tq, 0, t, bh, &sm->full[s]);
                    tma_load_3d(st + 24576, &p.tq, 64, t, bh, &sm->full[s]);
                }
                tma_load_3d(st + 32768, &p.tv, 0, t, bh, &sm->full[s]);
                tma_load_3d(st + 40960, &p.tv, 64, t, bh, &sm->full[s]);
                issued[s] = u + 1;
            }
            for (int s = 0; s < NST; ++s)
                if (issued[s] > 0) drain_wait(&sm->full[s], (issued[s] - 1) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t sbf = sb + Y::kSbf;
            const uint32_t id_g = idesc_bf16(64, 64, false, false);
            const uint32_t id_o1 = idesc_bf16(64, 128, false, false);
            const uint32_t id_o2 = idesc_bf16(64, 128, false, true);
            const uint32_t id_ds = idesc_bf16(128, 128, true, true);
            if (kOut) {
                // G(j) = phi(Q) phi(K)^T or Q K^T of chunk j, into G[j & 1]
                auto take = [&](int j) -> bool {
                    const int s = j % NST, u = j / NST;
                    if (!mbar_wait(&sm->full[s], u & 1, abort, p.err)) return false;
                    if (!mbar_wait(&sm->prep_done[s], u & 1, abort, p.err)) return false;
                    tc_fence_after();
                    const uint32_t st = sb + s * Y::kStage;
                    mma_chain<8, true, true>(tm + kColG01 + 64 * (j & 1), dk(st + 8192), dk(st), id_g, false);
                    mma_commit(&sm->g_done[j & 1]);
                    return true;
                };
                bool ok = take(0);
                for (int c = 0; c < nch && ok; ++c) {
                    const int s = c % NST;
                    const uint32_t st = sb + s * Y::kStage;
                    const uint32_t at = sb + Y::kA + (c & 1) * 8192;
                    if (c + 1 < nch && !take(c + 1)) break;
                    if (!mbar_wait(&sm->a_ready[c & 1], (c >> 1) & 1, abort, p.err)) break;
                    if (!mbar_wait(&sm->s_ready, c & 1, abort, p.err)) break;
                    tc_fence_after();
                    mma_chain<8, true, true>(tm + kColP01, dk(st + 8192), dk(sbf), id_o1, false);   // Q S^T
                    mma_chain<4, true, false>(tm + kColO01, dk(at), dmn(st + 32768, 8192), id_o2,
                                              false);                                             // A V
                    mma_chain<4, false, false>(tm + kColDS, dmn(st + 32768, 8192), dmn(st, 16384), id_ds,
                                               false);                                          // dS = V^T K~
                    mma_commit(&sm->mma2_done);
                    mma_commit(&sm->empty[s]);
                }
            } else {
                for (int c = 0; c < nch; ++c) {
                    const int s = c % NST, u = c / NST, b = c & 1;
                    const uint32_t st = sb + s * Y::kStage;
                    if (!mbar_wait(&sm->full[s], u & 1, abort, p.err)) break;
                    if (!mbar_wait(&sm->prep_done[s], u & 1, abort, p.err)) break;
                    if (c >= 2 && !mbar_wait(&sm->ds_free[b], ((c >> 1) - 1) & 1, abort, p.err)) break;
                    tc_fence_after();
                    mma_chain<4, false, false>(tm + kColDS + 128 * b, dmn(st + 32768, 8192), dmn(st, 16384),
                                               id_ds, false);
                    mma_commit(&sm->ds_done[b]);
                    mma_commit(&sm->empty[s]);
                }
            }
            mma_commit(&sm->fin);
            drain_wait(&sm->fin, 0);
        }
    } else if (warp >= 10) {
        // ------------------------------------------------------------ chunk preparation
        const int pe = threadIdx.x - 320;      // 0..63
        const int pw = pe >> 5;
        float gsum = 0.f;
        const bool gated = p.gate != nullptr;
        float graw = gated ? ld_gate(p, bh, tb, min(kC, te - tb), pe) : 1.f;
        for (int j = 0; j < nch; ++j) {
            const int s = j % NST, u = j / NST;
            const int t0 = tb + kC * j;
            const int L = min(kC, te - t0);
            float gnext = 1.f;
            if (gated && j + 1 < nch) gnext = ld_gate(p, bh, t0 + kC, min(kC, te - t0 - kC), pe);
            {
                float g = (gated && pe < L) ? lg2(fmaxf(graw, FLT_MIN)) : 0.f;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float n = __shfl_up_sync(0xffffffffu, g, off);
                    if (lane >= off) g += n;
                }
                if (lane == 31) sm->scan_tmp[pw] = g;
                named_sync(2, 64);
                if (pw == 1) g += sm->scan_tmp[0];
                sm->lam[j & 7][pe] = g;
                if (pe == kC - 1) gsum += g;
            }
            if (pe == 0) sm->len[j & 7] = L;
            bool ok = true;
            if (pe == 0) ok = mbar_wait(&sm->full[s], u & 1, abort, p.err);
            if (named_sync_any(2, 64, !ok)) break;
            const uint32_t st = sb + s * Y::kStage;
            if (!kOut) {
                // LOCAL pass: K~ = diag(dec) K in place, dec_r = 2^(lam_{C-1} - lam_r)
                named_sync(2, 64);   // the whole prefix is written
                const float *lam = sm->lam[j & 7];
                const float lamL = lam[kC - 1];
#pragma unroll
                for (int i4 = 0; i4 < 16; i4 += 4) {
                    uint4 w[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int n = pe + 64 * (i4 + i);
                        w[i] = lds128(st + (n >> 9) * 16384 + (n & 511) * 16);
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int n = pe + 64 * (i4 + i);
                        const int r = (n & 511) >> 3;
                        sts128(st + (n >> 9) * 16384 + (n & 511) * 16,
                               scale_bf16x8(w[i], r < L ? ex2(lamL - lam[r]) : 0.f));
                    }
                }
            }
            fence_async_smem();
            named_sync(2, 64);
            if (pe == 0) mbar_arrive(&sm->prep_done[s]);
            graw = gnext;
        }
        if (!kOut && pe == kC - 1 && p.gam_out)
            p.gam_out[(size_t)seg * p.BH + bh] = ex2(gsum);
    } else {
        // ------------------------------------------------------------ epilogue warps 2-9
        const int e = threadIdx.x - 64;        // 0..255
        const int q = warp & 3;                // TMEM lane quarter of this warp
        const int h = (warp - 2) >> 2;         // column half
        const int row = 32 * q + lane;         // M=128 accumulator row = state row
        const uint32_t tl = tm + ((uint32_t)(32 * q) << 16);
        const uint32_t sbf = sb + Y::kSbf;
        // M=64 accumulators: row 16 q + (lane & 15); lanes 16-31 take the second column range
        const int r64 = 16 * q + (lane & 15);
        const int hi = lane >> 4;

        float Sr[64];
        {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                float v[16];
                start_state16(p, seg, bh, row, 64 * h + 16 * g, v);
#pragma unroll
                for (int k = 0; k < 16; ++k) Sr[16 * g + k] = v[k];
            }
            if (kOut) {
#pragma unroll
                for (int g = 0; g < 4; ++g) st_row_bf16x16(sbf + h * 16384, row, 2 * g, Sr + 16 * g);
                fence_async_smem();
                epi_sync();
                if (e == 0) mbar_arrive(&sm->s_ready);
            }
        }

        if (kOut) {
            // A tile of chunk j from G(j): masks, decays (mode 1) or denominators (mode 0);
            // mode 1 also scales K to K~ = diag(dec) K once G(j) has consumed it.
            auto aepi = [&](int j) -> bool {
                const int s = j % NST, u = j / NST;
                bool ok = true;
                if (e == 0) {
                    ok = mbar_wait(&sm->prep_done[s], u & 1, abort, p.err) &&
                         mbar_wait(&sm->g_done[j & 1], (j >> 1) & 1, abort, p.err);
                    if (ok) ok = mbar_wait(&sm->full[s], u & 1, abort, p.err);
                }
                if (named_sync_any(1, kEpi, !ok)) return false;
                tc_fence_after();
                const int L = sm->len[j & 7];
                const float *lam = sm->lam[j & 7];
                const int i = r64;
                float v[16];
                tmem_ld_pair16(tl + kColG01 + 64 * (j & 1) + 32 * h, v);
                const int c0 = 32 * h + 16 * hi;
                const float li = lam[i];
#pragma unroll
                for (int k = 0; k < 16; ++k) v[k] = (c0 + k <= i) ? v[k] * ex2(li - lam[c0 + k]) : 0.f;
                st_row_bf16x16(sb + Y::kA + (j & 1) * 8192, i, c0 >> 3, v);
                {   // K <- diag(dec) K in place, now that G(j) has consumed K
                    const uint32_t st = sb + s * Y::kStage;
                    const float lamL = lam[kC - 1];
                    uint4 w[4];
#pragma unroll
                    for (int it = 0; it < 4; ++it) {
                        const int n = e + kEpi * it;
                        w[it] = lds128(st + (n >> 9) * 16384 + (n & 511) * 16);
                    }
#pragma unroll
                    for (int it = 0; it < 4; ++it) {
                        const int n = e + kEpi * it;
                        const int r = (n & 511) >> 3;
                        sts128(st + (n >> 9) * 16384 + (n & 511) * 16,
                               scale_bf16x8(w[it], r < L ? ex2(lamL - lam[r]) : 0.f));
                    }
                }
                fence_async_smem();
                tc_fence_before();
                epi_sync();
                if (e == 0) {
                    mbar_arrive(&sm->a_ready[j & 1]);
                    mbar_arrive(&sm->empty[s]);   // the epilogue is done with this stage
                }
                return true;
            };

            bool ok = aepi(0);
            for (int c = 0; c < nch && ok; ++c) {
                const int t0 = tb + kC * c;
                if (c + 1 < nch && !aepi(c + 1)) break;
                bool w_ok = true;
                if (e == 0) {
                    w_ok = mbar_wait(&sm->mma2_done, c & 1, abort, p.err);
                    tma_store_wait_read<0>();   // output staging free again
                }
                if (named_sync_any(1, kEpi, !w_ok)) break;
                tc_fence_after();
                const int L = sm->len[c & 7];
                const float *lam = sm->lam[c & 7];
                // ---- outputs of chunk c: row t = r64, columns 64 h + 32 hi + [0, 32)
                const bool direct = p.cu && L < kC;   // partial chunk of a packed sequence
                {
                    const int t = r64;
                    const bool has = t < L;
                    const float scale = has ? ex2(lam[t]) : 1.f;
                    float v[32], pq[32];
                    tmem_ld_pair32(tl + kColO01 + 64 * h, v);
                    tmem_ld_pair32(tl + kColP01 + 64 * h, pq);
#pragma unroll
                    for (int k = 0; k < 32; ++k) v[k] = fmaf(scale, pq[k], v[k]);
                    if (has && direct) {
                        st_out_row32(p, bh, t0 + t, 64 * h + 32 * hi, v);
                    } else if (has) {
                        const uint32_t ost = sb + Y::kOst + h * 8192;
                        st_row_bf16x16(ost, t, 4 * hi, v);
                        st_row_bf16x16(ost, t, 4 * hi + 2, v + 16);
                    }
                }
                // ---- state: S <- g S + dS (registers), bf16 copy for the next products
                const bool last = (c + 1 == nch);
                {
                    const float gC = ex2(lam[kC - 1]);
                    float v[64];
                    tmem_ld64(tl + kColDS + 64 * h, v);
#pragma unroll
                    for (int k = 0; k < 64; ++k) Sr[k] = fmaf(gC, Sr[k], v[k]);
                    if (!last) {
#pragma unroll
                        for (int g = 0; g < 4; ++g)
                            st_row_bf16x16(sbf + h * 16384, row, 2 * g, Sr + 16 * g);
                    }
                }
                fence_async_smem();
                tc_fence_before();
                epi_sync();
                if (e == 0) {
                    mbar_arrive(&sm->s_ready);
                    if (!direct) {
                        tma_store_3d(&p.to, sb + Y::kOst, 0, t0, bh);
                        tma_store_3d(&p.to, sb + Y::kOst + 8192, 64, t0, bh);
                        tma_store_commit();
                    }
                }
                if (last && p.s_out && (!p.out_last_only || seg == p.nseg - 1)) {
                    float *dst = p.s_out + (size_t)seg * p.s_out_seg + (size_t)bh * kD * kD +
                                 (size_t)row * kD + 64 * h;
#pragma unroll
                    for (int k = 0; k < 64; k += 4)
                        *reinterpret_cast<float4 *>(dst + k) =
                            make_float4(Sr[k], Sr[k + 1], Sr[k + 2], Sr[k + 3]);
                }
            }
            if (e == 0) tma_store_wait_all<0>();
        } else {
            for (int c = 0; c < nch; ++c) {
                const int s = c % NST, u = c / NST, b = c & 1;
                bool ok = true;
                if (e == 0)
                    ok = mbar_wait(&sm->prep_done[s], u & 1, abort, p.err) &&
                         mbar_wait(&sm->ds_done[b], (c >> 1) & 1, abort, p.err);
                if (e == 0 && ok) mbar_arrive(&sm->empty[s]);   // stage: only dS(c) reads it
                if (named_sync_any(1, kEpi, !ok)) break;
                tc_fence_after();
                const float gC = ex2(sm->lam[c & 7][kC - 1]);
                float v[64];
                tmem_ld64(tl + kColDS + 128 * b + 64 * h, v);
#pragma unroll
                for (int k = 0; k < 64; ++k) Sr[k] = fmaf(gC, Sr[k], v[k]);
                tc_fence_before();
                epi_sync();
                if (e == 0) mbar_arrive(&sm->ds_free[b]);
                if (c + 1 == nch && p.s_out) {
                    float *dst = p.s_out + (size_t)seg * p.s_out_seg + (size_t)bh * kD * kD +
                                 (size_t)row * kD + 64 * h;
#pragma unroll
                    for (int k = 0; k < 64; k += 4)
                        *reinterpret_cast<float4 *>(dst + k) =
                            make_float4(Sr[k], Sr[k + 1], Sr[k + 2], Sr[k + 3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tm, kTmemCols);
    }
}

// ------------------------------------------------------------------ mode 0
// elu(x)+1 linear attention with the z normaliser.  No gate acts on the state, so the
// fp32 state lives in tensor memory and each chunk's dS = V^T phi(K) is accumulated into
// it by the MMA itself.  What remains per chunk is dominated by the feature map: 2 x 64 x
// 128 exponentials, which the special-function units deliver at 16 per clock per SM.
// Eight preparation warps, two on each SM sub-partition, share that work.  18 warps:
//   warp 0      TMA producer,
//   warp 1      owns TMEM; lane 0 issues every MMA,
//   warps 2-9   epilogue: A tile and denominators, bf16 copy of the state, outputs,
//   warps 10-17 preparation: phi applied in place to the Q and K tiles, the running
//               column sums z, and phi(q_t) . z_{chunk start}.
// TMEM: S 0-127 (M=128), G = phi(Q) phi(K)^T 128-255 (two M=64 buffers), O 256-511 (two
// M=64 buffers, so that the outputs of chunk c are read while chunk c+1 is computed).
// Shared memory holds two rings filled by TMA: K and Q tiles, four deep, because the
// preparation warps and Q K^T need them early; V tiles, two deep, needed only by the
// products of the chunk.  The outputs of a chunk are staged in its own V slot, dead once
// the products are done, and written by TMA; that slot is released when the store has read
// it, while the K/Q slot is released as soon as the products and the A-epilogue are done.  G is formed two chunks ahead, after the products of the
// current chunk, so that the tensor core runs the state chain products(c) -> state copy
// -> products(c+1) without waiting behind it.
// The tensor core commits once after Q S^T and dS (the epilogue may then copy the new
// state) and once after A V (the outputs are complete).
constexpr int kThreadsE = 576;
constexpr int kPrepE = 256;   // preparation threads (warps 10-17)
constexpr uint32_t kColSE = 0, kColGE = 128, kColOE = 256;

struct SmallE {
    uint64_t full_kq[4], empty_kq[4], prep_done[4], full_v[2], empty_v[2];
    uint64_t g_done[2], a_ready[2], o_free[2], mma2_done[2];
    uint64_t s_ready, s_done, fin;
    uint32_t tmem_base;
    int abort;
    int len[8];
    float part[8][4][kC];        // denominators: A row-sum halves [0, 1], phi(q).z halves [2, 3]
    alignas(16) float zsm[kD];   // z after the previous chunk (float4 reads)
    float zpart[8][64];          // per-warp column sums of phi(K)
};
struct LayE {
    static constexpr int kKQStages = 4, kVStages = 2;
    static constexpr uint32_t kKQ = 0;                      // 4 x 32 KB [K0][Q0][K1][Q1], 8 KB each
    static constexpr uint32_t kV = kKQ + kKQStages * 32768;  // 2 x 16 KB [V0][V1]
    static constexpr uint32_t kSbf = kV + kVStages * 16384;  // 32 KB bf16 state [d_v][d_k]
    static constexpr uint32_t kA = kSbf + 32768;             // 2 x 8 KB A tiles [t][j]
    static constexpr uint32_t kSmall = kA + 16384;
    static constexpr uint32_t kBytes = kSmall + sizeof(SmallE);
};
static_assert(LayE::kBytes <= 227 * 1024, "shared memory per CTA");

__device__ __forceinline__ void phi_bf16x8(uint4 &w) {
    w.x = phi_bf16x2(w.x);
    w.y = phi_bf16x2(w.y);
    w.z = phi_bf16x2(w.z);
    w.w = phi_bf16x2(w.w);
}

template <int KIND>
__global__ void __launch_bounds__(kThreadsE, 1) prefill_elu_kernel(const __grid_constant__ TcParams p) {
    using Y = LayE;
    constexpr int NKQ = Y::kKQStages, NV = Y::kVStages;
    constexpr bool kOut = (KIND == kOutput);
    static_assert(KIND == kOutput || KIND == kLocal, "output or local pass");

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sb = smem_u32(smem_raw);
    if (sb & 1023u) {
        if (threadIdx.x == 0 && p.err) atomicOr(p.err, (unsigned)kErrBadLaunch);
        return;
    }
    SmallE *sm = reinterpret_cast<SmallE *>(smem_raw + Y::kSmall);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const CtaRange rng = cta_range<false>(p, (int)blockIdx.x);
    const int bh = rng.bh, seg = rng.seg, tb = rng.tb, te = rng.te;
    if (te <= tb) return;   // an empty packed sequence: nothing to read or write
    const int nch = (te - tb + kC - 1) / kC;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NKQ; ++s) {
            mbar_init(&sm->full_kq[s], 1);
            mbar_init(&sm->empty_kq[s], kOut ? 2 : 1);   // tensor core (+ A-epilogue)
            mbar_init(&sm->prep_done[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm->full_v[b], 1);
            mbar_init(&sm->empty_v[b], kOut ? 2 : 1);   // tensor core (+ output store)
            mbar_init(&sm->g_done[b], 1);
            mbar_init(&sm->a_ready[b], 1);
            mbar_init(&sm->o_free[b], 1);
            mbar_init(&sm->mma2_done[b], 1);
        }
        mbar_init(&sm->s_ready, 1);
        mbar_init(&sm->s_done, 1);
        mbar_init(&sm->fin, 1);
        sm->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = sm->tmem_base;
    volatile int *abort = &sm->abort;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        // Both rings are refilled as soon as their slot is released, whichever comes
        // first: the K/Q ring runs up to four chunks ahead, the V ring two.
        if (lane == 0) {
            tma_prefetch_desc(&p.tk);
            tma_prefetch_desc(&p.tv);
            if (kOut) tma_prefetch_desc(&p.tq);
            int nkq = 0, nv = 0;
            uint32_t idle = 0;
            while ((nkq < nch || nv < nch) && !*abort) {
                bool moved = false;
                if (nkq < nch && (nkq < NKQ || mbar_try_wait(&sm->empty_kq[nkq % NKQ], ((nkq / NKQ) - 1) & 1))) {
                    const int s = nkq % NKQ, t = tb + kC * nkq;
                    const uint32_t st = sb + Y::kKQ + s * 32768;
                    mbar_arrive_expect_tx(&sm->full_kq[s], kOut ? 32768u : 16384u);
                    tma_load_3d(st + 0, &p.tk, 0, t, bh, &sm->full_kq[s]);
                    tma_load_3d(st + 16384, &p.tk, 64, t, bh, &sm->full_kq[s]);
                    if (kOut) {
                        tma_load_3d(st + 8192, &p.tq, 0, t, bh, &sm->full_kq[s]);
                        tma_load_3d(st + 24576, &p.tq, 64, t, bh, &sm->full_kq[s]);
                    }
                    ++nkq;
                    moved = true;
                }
                if (nv < nch && (nv < NV || mbar_try_wait(&sm->empty_v[nv % NV], ((nv / NV) - 1) & 1))) {
                    const int s = nv % NV, t = tb + kC * nv;
                    const uint32_t sv = sb + Y::kV + s * 16384;
                    mbar_arrive_expect_tx(&sm->full_v[s], 16384u);
                    tma_load_3d(sv + 0, &p.tv, 0, t, bh, &sm->full_v[s]);
                    tma_load_3d(sv + 8192, &p.tv, 64, t, bh, &sm->full_v[s]);
                    ++nv;
                    moved = true;
                }
                if (moved) {
                    idle = 0;
                } else if (++idle > kSpinLimit) {
                    *abort = 1;
                    if (p.err) atomicOr(p.err, 1u);
                }
            }
            // wait for the copies in flight before the CTA may exit
            for (int c = max(0, nkq - NKQ); c < nkq; ++c) drain_wait(&sm->full_kq[c % NKQ], (c / NKQ) & 1);
            for (int c = max(0, nv - NV); c < nv; ++c) drain_wait(&sm->full_v[c % NV], (c / NV) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t sbf = sb + Y::kSbf;
            const uint32_t id_g = idesc_bf16(64, 64, false, false);
            const uint32_t id_o1 = idesc_bf16(64, 128, false, false);
            const uint32_t id_o2 = idesc_bf16(64, 128, false, true);
            const uint32_t id_ds = idesc_bf16(128, 128, true, true);
            if (kOut) {
                auto take = [&](int j) -> bool {   // G(j) = phi(Q) phi(K)^T into G[j & 1]
                    const int s = j % NKQ, u = j / NKQ;
                    if (!mbar_wait(&sm->full_kq[s], u & 1, abort, p.err)) return false;
                    if (!mbar_wait(&sm->prep_done[s], u & 1, abort, p.err)) return false;
                    tc_fence_after();
                    const uint32_t st = sb + Y::kKQ + s * 32768;
                    mma_chain<8, true, true>(tm + kColGE + 64 * (j & 1), dk(st + 8192), dk(st), id_g, false);
                    mma_commit(&sm->g_done[j & 1]);
                    return true;
                };
                bool ok = take(0) && (nch < 2 || take(1));
                for (int c = 0; c < nch && ok; ++c) {
                    const int s = c % NKQ, b = c & 1, sv = c % NV;
                    const uint32_t st = sb + Y::kKQ + s * 32768;
                    const uint32_t vt = sb + Y::kV + sv * 16384;
                    const uint32_t at = sb + Y::kA + b * 8192;
                    const uint32_t to = tm + kColOE + 128 * b;
                    if (!mbar_wait(&sm->a_ready[b], (c >> 1) & 1, abort, p.err)) break;
                    if (!mbar_wait(&sm->s_ready, c & 1, abort, p.err)) break;
                    if (c >= 2 && !mbar_wait(&sm->o_free[b], ((c >> 1) - 1) & 1, abort, p.err)) break;
                    if (!mbar_wait(&sm->full_v[sv], (c / NV) & 1, abort, p.err)) break;
                    tc_fence_after();
                    mma_chain<8, true, true>(to, dk(st + 8192), dk(sbf), id_o1, false);      // phi(Q) S^T
                    mma_chain<4, false, false>(tm + kColSE, dmn(vt, 8192), dmn(st, 16384), id_ds,
                                               true);                                     // S += V^T phi(K)
                    mma_commit(&sm->s_done);
                    mma_chain<4, true, false>(to, dk(at), dmn(vt, 8192), id_o2, true);      // + A V
                    mma_commit(&sm->mma2_done[b]);
                    mma_commit(&sm->empty_kq[s]);
                    mma_commit(&sm->empty_v[sv]);
                    if (c + 2 < nch && !take(c + 2)) break;
                }
            } else {
                bool ok = mbar_wait(&sm->s_ready, 0, abort, p.err);   // initial state in TMEM
                for (int c = 0; c < nch && ok; ++c) {
                    const int s = c % NKQ, u = c / NKQ, sv = c % NV;
                    const uint32_t st = sb + Y::kKQ + s * 32768;
                    const uint32_t vt = sb + Y::kV + sv * 16384;
                    if (!mbar_wait(&sm->full_kq[s], u & 1, abort, p.err)) break;
                    if (!mbar_wait(&sm->prep_done[s], u & 1, abort, p.err)) break;
                    if (!mbar_wait(&sm->full_v[sv], (c / NV) & 1, abort, p.err)) break;
                    tc_fence_after();
                    mma_chain<4, false, false>(tm + kColSE, dmn(vt, 8192), dmn(st, 16384), id_ds, true);
                    mma_commit(&sm->empty_kq[s]);
                    mma_commit(&sm->empty_v[sv]);
                }
                mma_commit(&sm->s_done);
            }
            mma_commit(&sm->fin);
            drain_wait(&sm->fin, 0);
        }
    } else if (warp >= 10) {
        // ------------------------------------------------------------ preparation
        const int pe = threadIdx.x - 320;      // 0..255
        const int pw = pe >> 5;                // 0..7
        const int ch = lane & 7, rg = lane >> 3;
        float zc = 0.f;                        // z of column pe (pe < 128)
        if (pe < kD) {
            zc = start_z(p, seg, bh, pe);
            sm->zsm[pe] = zc;
        }
        // Warp pw takes column half pw >> 2 and rows 16 (pw & 3) + 4 rg + i (i < 4); lane
        // chunk ch holds columns 8 ch .. 8 ch + 7 of that half.
        const int hw = pw >> 2;
        const uint32_t half = (uint32_t)hw * 16384;
        const int r0 = 16 * (pw & 3) + 4 * rg;
        for (int j = 0; j < nch; ++j) {
            const int s = j % NKQ, u = j / NKQ;
            const int L = min(kC, te - (tb + kC * j));
            if (pe == 0) sm->len[j & 7] = L;
            bool ok = true;
            if (pe == 0) ok = mbar_wait(&sm->full_kq[s], u & 1, abort, p.err);
            if (named_sync_any(2, kPrepE, !ok)) break;
            const uint32_t st = sb + Y::kKQ + s * 32768;
            if (kOut) {
                // phi(Q) in place, and phi(q_r) . z_{j-1} over this half (shuffle-reduced)
                const uint32_t qb = st + 8192 + half;
                const float4 za = *reinterpret_cast<const float4 *>(&sm->zsm[64 * hw + 8 * ch]);
                const float4 zb = *reinterpret_cast<const float4 *>(&sm->zsm[64 * hw + 8 * ch + 4]);
                uint4 w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) w[i] = lds128(qb + sw128_off(r0 + i, ch));
                float d[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    phi_bf16x8(w[i]);
                    const float2 f0 = unpack_bf16x2(w[i].x), f1 = unpack_bf16x2(w[i].y);
                    const float2 f2 = unpack_bf16x2(w[i].z), f3 = unpack_bf16x2(w[i].w);
                    d[i] = fmaf(f0.x, za.x, fmaf(f0.y, za.y, fmaf(f1.x, za.z, f1.y * za.w))) +
                           fmaf(f2.x, zb.x, fmaf(f2.y, zb.y, fmaf(f3.x, zb.z, f3.y * zb.w)));
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) sts128(qb + sw128_off(r0 + i, ch), w[i]);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    d[i] += __shfl_xor_sync(0xffffffffu, d[i], 1);
                    d[i] += __shfl_xor_sync(0xffffffffu, d[i], 2);
                    d[i] += __shfl_xor_sync(0xffffffffu, d[i], 4);
                }
                if (ch == 0)
#pragma unroll
                    for (int i = 0; i < 4; ++i) sm->part[j & 7][2 + hw][r0 + i] = d[i];
            }
            // phi(K) in place (rows past the chunk end zeroed) and its column sums
            {
                const uint32_t kb = st + half;
                uint4 w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) w[i] = lds128(kb + sw128_off(r0 + i, ch));
                float cs[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) cs[k] = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (r0 + i < L)
                        phi_bf16x8(w[i]);
                    else
                        w[i] = make_uint4(0u, 0u, 0u, 0u);
                    const uint32_t *wd = reinterpret_cast<const uint32_t *>(&w[i]);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float2 f = unpack_bf16x2(wd[k]);
                        cs[2 * k] += f.x;
                        cs[2 * k + 1] += f.y;
                    }
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) sts128(kb + sw128_off(r0 + i, ch), w[i]);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    cs[k] += __shfl_xor_sync(0xffffffffu, cs[k], 8);
                    cs[k] += __shfl_xor_sync(0xffffffffu, cs[k], 16);
                }
                if (rg == 0)
#pragma unroll
                    for (int k = 0; k < 8; ++k) sm->zpart[pw][8 * ch + k] = cs[k];
            }
            named_sync(2, kPrepE);   // column sums ready; every read of z_{j-1} is done
            if (pe < kD) {
                const int w0 = 4 * (pe >> 6), cc = pe & 63;
                zc += (sm->zpart[w0][cc] + sm->zpart[w0 + 1][cc]) +
                      (sm->zpart[w0 + 2][cc] + sm->zpart[w0 + 3][cc]);
                sm->zsm[pe] = zc;
            }
            fence_async_smem();
            named_sync(2, kPrepE);
            if (pe == 0) mbar_arrive(&sm->prep_done[s]);
        }
        if (pe < kD && p.z_out && (!p.out_last_only || seg == p.nseg - 1))
            p.z_out[(size_t)seg * p.z_out_seg + (size_t)bh * kD + pe] = zc;
    } else {
        // ------------------------------------------------------------ epilogue warps 2-9
        const int e = threadIdx.x - 64;        // 0..255
        const int q = warp & 3;                // TMEM lane quarter of this warp
        const int h = (warp - 2) >> 2;         // column half
        const int row = 32 * q + lane;         // state row (d_v index) = TMEM lane
        const uint32_t tl = tm + ((uint32_t)(32 * q) << 16);
        const uint32_t sbf = sb + Y::kSbf;
        const int r64 = 16 * q + (lane & 15);  // M=64 accumulator row of this thread
        const int hi = lane >> 4;

        // initial state into TMEM (and its bf16 copy for the first Q S^T)
        {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                float v[16];
                start_state16(p, seg, bh, row, 64 * h + 16 * g, v);
                tmem_st16(tl + kColSE + 64 * h + 16 * g, v);
                if (kOut) st_row_bf16x16(sbf + h * 16384, row, 2 * g, v);
            }
            fence_async_smem();
            tc_fence_before();
            epi_sync();
            if (e == 0) mbar_arrive(&sm->s_ready);
        }

        if (kOut) {
            // A tile of chunk j from G(j), with its row sums for the denominators
            auto aepi = [&](int j) -> bool {
                const int s = j % NKQ, u = j / NKQ;
                bool ok = true;
                if (e == 0)
                    ok = mbar_wait(&sm->prep_done[s], u & 1, abort, p.err) &&
                         mbar_wait(&sm->g_done[j & 1], (j >> 1) & 1, abort, p.err);
                if (named_sync_any(1, kEpi, !ok)) return false;
                tc_fence_after();
                const int i = r64;
                float v[16];
                tmem_ld_pair16(tl + kColGE + 64 * (j & 1) + 32 * h, v);
                const int c0 = 32 * h + 16 * hi;
                // pack once to bf16 (the MMA operand) and sum the packed values, so that the
                // denominators use exactly the weights A V is formed with
                uint32_t pk[8];
                float rs = 0.f;
#pragma unroll
                for (int k = 0; k < 16; k += 2) {
                    const uint32_t w = pack_bf16x2((c0 + k <= i) ? v[k] : 0.f,
                                                   (c0 + k + 1 <= i) ? v[k + 1] : 0.f);
                    pk[k >> 1] = w;
                    const float2 f = unpack_bf16x2(w);
                    rs += f.x + f.y;
                }
                const uint32_t at = sb + Y::kA + (j & 1) * 8192;
                sts128(at + sw128_off(i, c0 >> 3), make_uint4(pk[0], pk[1], pk[2], pk[3]));
                sts128(at + sw128_off(i, (c0 >> 3) + 1), make_uint4(pk[4], pk[5], pk[6], pk[7]));
                rs += __shfl_xor_sync(0xffffffffu, rs, 16);
                if (hi == 0) sm->part[j & 7][h][i] = rs;
                fence_async_smem();
                tc_fence_before();
                epi_sync();
                if (e == 0) {
                    mbar_arrive(&sm->a_ready[j & 1]);
                    mbar_arrive(&sm->empty_kq[s]);   // the epilogue is done with this K/Q slot
                    if (j >= 2) {   // the outputs of chunk j-2, stored a whole A-epilogue ago,
                        tma_store_wait_read<0>();    // have left their V slot: refill it
                        mbar_arrive(&sm->empty_v[(j - 2) % NV]);
                    }
                }
                return true;
            };

            bool ok = aepi(0);
            for (int c = 0; c < nch && ok; ++c) {
                const int t0 = tb + kC * c;
                const int b = c & 1;
                const bool last = (c + 1 == nch);
                if (c + 1 < nch && !aepi(c + 1)) break;
                // ---- state after chunk c: bf16 copy for the next products
                bool w_ok = true;
                if (e == 0) w_ok = mbar_wait(&sm->s_done, c & 1, abort, p.err);
                if (named_sync_any(1, kEpi, !w_ok)) break;
                tc_fence_after();
#pragma unroll
                for (int sub = 0; sub < 2; ++sub) {
                    float v[32];
                    tmem_ld32(tl + kColSE + 64 * h + 32 * sub, v);
                    if (!last) {
                        st_row_bf16x16(sbf + h * 16384, row, 4 * sub, v);
                        st_row_bf16x16(sbf + h * 16384, row, 4 * sub + 2, v + 16);
                    } else if (p.s_out && (!p.out_last_only || seg == p.nseg - 1)) {
                        float *dst = p.s_out + (size_t)seg * p.s_out_seg + (size_t)bh * kD * kD +
                                     (size_t)row * kD + 64 * h + 32 * sub;
#pragma unroll
                        for (int k = 0; k < 32; k += 4)
                            *reinterpret_cast<float4 *>(dst + k) = make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
                    }
                }
                fence_async_smem();
                tc_fence_before();
                epi_sync();
                if (e == 0) mbar_arrive(&sm->s_ready);
                // ---- outputs of chunk c: row t = r64, columns 64 h + 32 hi + [0, 32)
                if (e == 0) {
                    w_ok = mbar_wait(&sm->mma2_done[b], (c >> 1) & 1, abort, p.err);
                    tma_store_wait_read<0>();   // (normally long done) before the next staging
                }
                if (named_sync_any(1, kEpi, !w_ok)) break;
                tc_fence_after();
                const bool direct = p.cu && sm->len[c & 7] < kC;   // partial packed chunk
                {
                    const int L = sm->len[c & 7];
                    const int t = r64;
                    const bool has = t < L;
                    float scale = 1.f;
                    if (has) {
                        const float (*pt)[kC] = sm->part[c & 7];
                        scale = 1.f / ((pt[0][t] + pt[1][t]) + (pt[2][t] + pt[3][t]));
                    }
                    float v[32];
                    tmem_ld_pair32(tl + kColOE + 128 * b + 64 * h, v);
#pragma unroll
                    for (int k = 0; k < 32; ++k) v[k] *= scale;
                    if (has && direct) {
                        st_out_row32(p, bh, t0 + t, 64 * h + 32 * hi, v);
                    } else if (has) {   // this chunk's V slot: [V0 | V1] -> [O0 | O1], 8 KB each
                        const uint32_t ost = sb + Y::kV + (c % NV) * 16384 + h * 8192;
                        st_row_bf16x16(ost, t, 4 * hi, v);
                        st_row_bf16x16(ost, t, 4 * hi + 2, v + 16);
                    }
                }
                fence_async_smem();
                tc_fence_before();
                epi_sync();
                if (e == 0) {
                    mbar_arrive(&sm->o_free[b]);
                    if (!direct) {
                        const uint32_t ost = sb + Y::kV + (c % NV) * 16384;
                        tma_store_3d(&p.to, ost, 0, t0, bh);
                        tma_store_3d(&p.to, ost + 8192, 64, t0, bh);
                        tma_store_commit();
                    }
                }
            }
            if (e == 0) tma_store_wait_all<0>();
        } else {
            bool ok = true;
            if (e == 0) ok = mbar_wait(&sm->s_done, 0, abort, p.err);
            if (!named_sync_any(1, kEpi, !ok)) {
                tc_fence_after();
                float v[64];
                tmem_ld64(tl + kColSE + 64 * h, v);
                if (p.s_out) {
                    float *dst = p.s_out + (size_t)seg * p.s_out_seg + (size_t)bh * kD * kD +
                                 (size_t)row * kD + 64 * h;
#pragma unroll
                    for (int k = 0; k < 64; k += 4)
                        *reinterpret_cast<float4 *>(dst + k) = make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tm, kTmemCols);
    }
}

// ------------------------------------------------------------------ combine kernels
// modes 0/1: the local pass ran on `f` sub-segments per segment; their local states fold
// in order into the segment starts, S <- gam_j S + N_j (z <- z + zN_j), and after every
// f-th sub-segment the start of the next segment is written.  float4 per thread.
__global__ void combine_scalar_kernel(int BH, int nseg, int f, const float *s_init,
                                      const float *z_init, const float *nloc, const float *zloc,
                                      const float *gam, float *sst, float *zst, int mode) {
    const size_t per4 = (size_t)kD * kD / 4;
    const size_t total4 = (size_t)BH * per4;
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int nsub = (nseg - 1) * f;
    if (idx < total4) {
        const int bh = (int)(idx / per4);
        float4 sv = s_init ? reinterpret_cast<const float4 *>(s_init)[idx] : make_float4(0.f, 0.f, 0.f, 0.f);
        reinterpret_cast<float4 *>(sst)[idx] = sv;
        for (int j = 0; j < nsub; ++j) {
            const float g = (mode == 1) ? gam[(size_t)j * BH + bh] : 1.f;
            const float4 n = reinterpret_cast<const float4 *>(nloc)[(size_t)j * total4 + idx];
            sv = make_float4(fmaf(g, sv.x, n.x), fmaf(g, sv.y, n.y), fmaf(g, sv.z, n.z), fmaf(g, sv.w, n.w));
            if ((j + 1) % f == 0) reinterpret_cast<float4 *>(sst)[(size_t)((j + 1) / f) * total4 + idx] = sv;
        }
    }
    if (mode == 0 && idx < (size_t)BH * kD) {
        float zv = z_init ? z_init[idx] : 0.f;
        zst[idx] = zv;
        for (int j = 0; j < nsub; ++j) {
            zv += zloc[(size_t)j * BH * kD + idx];
            if ((j + 1) % f == 0) zst[(size_t)((j + 1) / f) * BH * kD + idx] = zv;
        }
    }
}

// delta rule: S <- S M_j + N_j over the sub-segments j in order (f per segment), writing
// the start of segment s+1 after its f-th (row-parallel; 16 rows of S per CTA).
constexpr int kCombRows = 16;
__global__ void __launch_bounds__(256) combine_matrix_kernel(int BH, int nseg, int f,
                                                             const float *s_init,
                                                             const float *nloc, const float *mtr,
                                                             float *sst) {
    extern __shared__ float csm[];
    float *Ms = csm;                       // [128][128]
    float *Ss = Ms + kD * kD;              // [16][128]
    const int bh = blockIdx.x;
    const int r0 = blockIdx.y * kCombRows;
    const size_t per = (size_t)kD * kD;
    const size_t total = (size_t)BH * per;
    for (int i = threadIdx.x; i < kCombRows * kD; i += 256) {
        const size_t g = (size_t)bh * per + (size_t)r0 * kD + i;
        const float v = s_init ? s_init[g] : 0.f;
        Ss[i] = v;
        sst[g] = v;
    }
    const int nsub = (nseg - 1) * f;
    for (int s = 0; s < nsub; ++s) {
        __syncthreads();
        const float *Mg = mtr + (size_t)s * total + (size_t)bh * per;
        for (int i = threadIdx.x; i < kD * kD / 4; i += 256)
            reinterpret_cast<float4 *>(Ms)[i] = reinterpret_cast<const float4 *>(Mg)[i];
        __syncthreads();
        float acc[8];
        const int col = threadIdx.x & 127;
        const int rb = (threadIdx.x >> 7) * 8;
#pragma unroll
        for (int r = 0; r < 8; ++r) acc[r] = 0.f;
        for (int k = 0; k < kD; ++k) {
            const float m = Ms[k * kD + col];
#pragma unroll
            for (int r = 0; r < 8; ++r) acc[r] = fmaf(Ss[(rb + r) * kD + k], m, acc[r]);
        }
        __syncthreads();
        const float *Ng = nloc + (size_t)s * total + (size_t)bh * per;
        const bool boundary = (s + 1) % f == 0;
        float *dst = sst + (size_t)((s + 1) / f) * total + (size_t)bh * per;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const size_t g = (size_t)(r0 + rb + r) * kD + col;
            const float v = acc[r] + Ng[g];
            Ss[(rb + r) * kD + col] = v;
            if (boundary) dst[g] = v;
        }
    }
}

// ------------------------------------------------------------------ host side
struct Plan {
    int nseg, seg_len;
    int sub;   // modes 0/1: the local pass runs on `sub` equal sub-segments per segment
};

// The segment plan for BH heads of T tokens whose workspace fits max_ws bytes (without a
// segmented plan that fits: one outputs pass over whole sequences).
size_t workspace_floats(int mode, int BH, const struct Plan &pl);
Plan plan_for(int mode, int BH, int T, size_t max_ws = SIZE_MAX) {
    const int nchunks = (T + kC - 1) / kC;
    int nseg = 1;
    const int sms = 148;
    if (BH < sms) nseg = sms / BH;
    nseg = std::max(1, std::min(nseg, nchunks / 4));   // keep segments >= 4 chunks
    const int chunks_per_seg = (nchunks + nseg - 1) / nseg;
    Plan pl;
    pl.seg_len = chunks_per_seg * kC;
    pl.nseg = (T + pl.seg_len - 1) / pl.seg_len;
    // The local pass covers segments 0 .. nseg-2 only; split them further so that it too
    // fills the SMs (sub-segments of at least four chunks, dividing the segment evenly).
    pl.sub = 1;
    if (mode < 2 && pl.nseg > 1) {
        int f = sms / (BH * (pl.nseg - 1));
        while (f > 1 && (chunks_per_seg % f != 0 || chunks_per_seg / f < 4)) --f;
        pl.sub = std::max(1, f);
    }
    if (mode >= 2 && pl.nseg > 1) {
        // Delta rule: the local and transition CTAs of the segments 0 .. nseg-2 share one
        // launch.  Splitting segments into f sub-segments gives more, shorter CTAs; cost
        // ~ waves x chunks per sub-segment + the combine's matrix steps (about two chunks'
        // time each), with sub-segments of at least eight chunks that fit the workspace.
        double best = 0.0;
        for (int f = 1; f <= 8; f *= 2) {
            if (f > 1 && (chunks_per_seg % f != 0 || chunks_per_seg / f < 8)) break;
            Plan t = pl;
            t.sub = f;
            if (f > 1 && sizeof(float) * workspace_floats(mode, BH, t) > max_ws) break;
            const int ctas = 2 * BH * (pl.nseg - 1) * f;
            const double cost = (double)((ctas + sms - 1) / sms) * (chunks_per_seg / f) +
                                2.0 * (pl.nseg - 1) * f;
            if (f == 1 || cost < best) {
                best = cost;
                pl.sub = f;
            }
        }
    }
    if (pl.nseg > 1 && sizeof(float) * workspace_floats(mode, BH, pl) > max_ws) {
        pl.nseg = 1;
        pl.sub = 1;
        pl.seg_len = nchunks * kC;
    }
    return pl;
}

size_t workspace_floats(int mode, int BH, const Plan &pl) {
    if (pl.nseg <= 1) return 0;
    const size_t per = (size_t)BH * kD * kD;
    const size_t nloc = (size_t)(pl.nseg - 1) * pl.sub;   // local-pass sub-segments
    size_t f = (size_t)pl.nseg * per;                 // segment start states
    f += nloc * per;                                  // local states
    if (mode >= 2) f += nloc * per;                   // transitions (delta rule)
    if (mode == 1) f += nloc * BH;                    // gate products
    if (mode == 0) f += ((size_t)pl.nseg + nloc) * BH * kD;   // z starts + z locals
    return f;
}

template <int MODE, int KIND>
cudaError_t launch_kind(const TcParams &p, int grid, cudaStream_t stream) {
    cudaError_t e;
    if constexpr (MODE >= 2) {
        e = cudaFuncSetAttribute(prefill_tc_kernel<MODE, KIND>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, Lay<MODE>::kBytes);
        if (e != cudaSuccess) return e;
        timer_begin(stream);
        prefill_tc_kernel<MODE, KIND><<<grid, kThreads, Lay<MODE>::kBytes, stream>>>(p);
        timer_end(stream);
    } else {
        static_assert(KIND != kTransition && KIND != kLocalTrans,
                      "the transition pass belongs to the delta rule");
        if constexpr (MODE == 0) {
            e = cudaFuncSetAttribute(prefill_elu_kernel<KIND>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, LayE::kBytes);
            if (e != cudaSuccess) return e;
            timer_begin(stream);
            prefill_elu_kernel<KIND><<<grid, kThreadsE, LayE::kBytes, stream>>>(p);
            timer_end(stream);
        } else {
            e = cudaFuncSetAttribute(prefill01_kernel<MODE, KIND>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, Lay01::kBytes);
            if (e != cudaSuccess) return e;
            timer_begin(stream);
            prefill01_kernel<MODE, KIND><<<grid, kThreads01, Lay01::kBytes, stream>>>(p);
            timer_end(stream);
        }
    }
    note_launches(1);
    return cudaGetLastError();
}

template <int MODE>
cudaError_t run_mode(const PrefillArgs &a, const TcParams &base, const Plan &pl, float *ws) {
    const int BH = a.B * a.H;
    const size_t per = (size_t)BH * kD * kD;
    if (pl.nseg == 1) {
        TcParams p = base;
        p.s_in_mode = a.init_state ? 1 : 0;
        p.s_in = a.state;
        p.s_in_seg = 0;
        p.z_in = a.z;
        p.z_in_seg = 0;
        p.s_out = a.state;
        p.s_out_seg = 0;
        p.z_out = a.z;
        p.z_out_seg = 0;
        p.out_last_only = 1;
        return launch_kind<MODE, kOutput>(p, BH, a.stream);
    }
    const int nsub = (pl.nseg - 1) * pl.sub;                     // local-pass CTAs per head
    float *sst = ws;
    float *nloc = sst + (size_t)pl.nseg * per;
    float *mtr = nloc + (size_t)nsub * per;                      // mode 2 (sub = 1)
    float *gam = nloc + (size_t)nsub * per;                      // mode 1
    float *zst = nloc + (size_t)nsub * per;                      // mode 0
    float *zloc = zst + (size_t)pl.nseg * BH * kD;
    // pass A: local states of the sub-segments (and, delta rule, their transitions, in
    // the same launch)
    {
        TcParams p = base;
        p.s_in_mode = 0;
        p.s_out = nloc;
        p.s_out_seg = (long long)per;
        p.z_out = (MODE == 0) ? zloc : nullptr;
        p.z_out_seg = (long long)BH * kD;
        p.gam_out = (MODE == 1) ? gam : nullptr;
        p.out_last_only = 0;
        p.seg_len = pl.seg_len / pl.sub;
        p.nseg = nsub;
        cudaError_t e;
        if constexpr (MODE >= 2) {
            p.s_out2 = mtr;
            p.split = BH * nsub;
            e = launch_kind<MODE, kLocalTrans>(p, 2 * BH * nsub, a.stream);
        } else {
            e = launch_kind<MODE, kLocal>(p, BH * nsub, a.stream);
        }
        if (e != cudaSuccess) return e;
    }
    // Outputs pass.  Without an initial state and with few sub-segments per head, each
    // outputs CTA folds its own start state from the local states (no combine launch).
    // With an initial state the starts are first copied into the workspace by the combine
    // kernel: the outputs pass overwrites the caller's state with the final one.
    if constexpr (MODE < 2) {
        if (!a.init_state && nsub <= 4) {
            TcParams p = base;
            p.s_in_mode = 3;
            p.fold_init = nullptr;
            p.fold_zinit = nullptr;
            p.fold_loc = nloc;
            p.fold_zloc = (MODE == 0) ? zloc : nullptr;
            p.fold_gam = (MODE == 1) ? gam : nullptr;
            p.fold_sub = pl.sub;
            p.s_out = a.state;
            p.s_out_seg = 0;
            p.z_out = a.z;
            p.z_out_seg = 0;
            p.out_last_only = 1;
            return launch_kind<MODE, kOutput>(p, BH * pl.nseg, a.stream);
        }
    }
    // combine: segment start states
    const float *s_init = a.init_state ? a.state : nullptr;
    if constexpr (MODE >= 2) {
        const size_t bytes = sizeof(float) * (kD * kD + kCombRows * kD);
        cudaError_t e = cudaFuncSetAttribute(combine_matrix_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        if (e != cudaSuccess) return e;
        timer_begin(a.stream);
        combine_matrix_kernel<<<dim3(BH, kD / kCombRows), 256, bytes, a.stream>>>(
            BH, pl.nseg, pl.sub, s_init, nloc, mtr, sst);
        timer_end(a.stream);
    } else {
        const size_t total4 = per / 4;
        timer_begin(a.stream);
        combine_scalar_kernel<<<(unsigned)((total4 + 255) / 256), 256, 0, a.stream>>>(
            BH, pl.nseg, pl.sub, s_init, (MODE == 0 && a.init_state) ? a.z : nullptr, nloc, zloc, gam,
            sst, zst, MODE);
        timer_end(a.stream);
    }
    note_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // pass C: outputs from the exact segment starts
    TcParams p = base;
    p.s_in_mode = 1;
    p.s_in = sst;
    p.s_in_seg = (long long)per;
    p.z_in = (MODE == 0) ? zst : nullptr;
    p.z_in_seg = (long long)BH * kD;
    p.s_out = a.state;
    p.s_out_seg = 0;
    p.z_out = a.z;
    p.z_out_seg = 0;
    p.out_last_only = 1;
    return launch_kind<MODE, kOutput>(p, BH * pl.nseg, a.stream);
}

}  // namespace

bool prefill_tc_supports(int mode, int dtype, int dk, int dv, int chunk) {
    // modes 0-3 in bf16 with d = 128 at chunk 64 (chunk 32 selects the CUDA-core path,
    // which in mode 3 is exact for every gate value: no clamp)
    return dtype == LA_BF16 && dk == kD && dv == kD &&
           (chunk == 0 || chunk == kC);
}

size_t prefill_tc_workspace_bytes(int mode, int B, int H, int T, bool minimal) {
    const int BH = B * H;
    if (prefill_gdn_selected(mode, BH, false)) return minimal ? 0 : prefill_gdn_workspace_bytes(BH, T);
    if (!minimal && prefill_kda2_selected(mode, BH, false)) return prefill_kda2_workspace_bytes(BH, T);
    Plan pl = plan_for(mode, BH, T);
    if (minimal && mode >= 2) pl.sub = 1;   // the smallest segmented plan
    return sizeof(float) * workspace_floats(mode, BH, pl);
}

// Packed sequences: one outputs-pass CTA per (sequence, head), started from the
// sequence's own state slot (or zero) and writing its final state there.
template <int MODE>
cudaError_t run_packed(const PrefillArgs &a, const TcParams &base) {
    TcParams p = base;
    p.cu = a.cu;
    p.nseg = a.nseq;
    p.s_in_mode = a.init_state ? 1 : 0;
    p.s_in = a.state;
    p.s_in_seg = (long long)a.H * kD * kD;
    p.z_in = a.z;
    p.z_in_seg = (long long)a.H * kD;
    p.s_out = a.state;
    p.s_out_seg = (long long)a.H * kD * kD;
    p.z_out = a.z;
    p.z_out_seg = (long long)a.H * kD;
    p.out_last_only = 0;
    return launch_kind<MODE, kOutput>(p, a.nseq * a.H, a.stream);
}

cudaError_t launch_prefill_tc(const PrefillArgs &a, void *workspace, size_t workspace_bytes) {
    const int BH = a.B * a.H;
    if (prefill_gdn_selected(a.mode, BH, a.cu != nullptr)) return launch_prefill_gdn(a, workspace, workspace_bytes);
    // KDA with room for the per-chunk records (and gates the bulk copies can read): the
    // two-pass chain kernel; otherwise the segmented kernels with what the workspace allows
    if (prefill_kda2_selected(a.mode, BH, a.cu != nullptr) && workspace &&
        workspace_bytes >= prefill_kda2_workspace_bytes(BH, a.T) &&
        (reinterpret_cast<uintptr_t>(workspace) & 15u) == 0 && (reinterpret_cast<uintptr_t>(a.gate) & 15u) == 0)
        return launch_prefill_kda2(a, workspace, workspace_bytes);
    const Plan pl = plan_for(a.mode, BH, a.T, workspace ? workspace_bytes : 0);
    TcParams p;
    memset(&p, 0, sizeof(p));
    const uint64_t row_pitch = kD * 2, head_pitch = (uint64_t)a.T * kD * 2;
    if (!make_tmap_3d(&p.tq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kD, a.T, BH, row_pitch,
                      head_pitch, 64, kC, true) ||
        !make_tmap_3d(&p.tk, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kD, a.T, BH, row_pitch,
                      head_pitch, 64, kC, true) ||
        !make_tmap_3d(&p.tv, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kD, a.T, BH, row_pitch,
                      head_pitch, 64, kC, true) ||
        !make_tmap_3d(&p.to, a.o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kD, a.T, BH, row_pitch,
                      head_pitch, 64, kC, true))
        return cudaErrorInvalidValue;
    p.gate = a.gate;
    p.gate_heads = a.gate_heads;
    p.beta = a.beta;
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.T = a.T;
    p.BH = BH;
    p.seg_len = pl.seg_len;
    p.nseg = pl.nseg;
    p.err = device_error_word();
    float *ws = static_cast<float *>(workspace);
    if (a.cu) {
        switch (a.mode) {
            case LA_MODE_ELU1_NORM: return run_packed<0>(a, p);
            case LA_MODE_GATED: return run_packed<1>(a, p);
            case LA_MODE_GATED_DELTA: return run_packed<2>(a, p);
            case LA_MODE_KDA: return run_packed<3>(a, p);
        }
        return cudaErrorInvalidValue;
    }
    switch (a.mode) {
        case LA_MODE_ELU1_NORM: return run_mode<0>(a, p, pl, ws);
        case LA_MODE_GATED: return run_mode<1>(a, p, pl, ws);
        case LA_MODE_GATED_DELTA: return run_mode<2>(a, p, pl, ws);
        case LA_MODE_KDA: return run_mode<3>(a, p, pl, ws);
    }
    return cudaErrorInvalidValue;
}

}  // namespace la

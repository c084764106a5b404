// prefill_gdn.cu -- single-pass chunked prefill of the gated delta rule (mode 2) on the
// 5th-generation tensor cores, bf16 I/O, d_k = d_v = 128, chunk C = 64, fp32 state.
//
// The update is the Gated DeltaNet equation of the lesson page "Linear attention and
// hybrids", section "The delta rule and Gated DeltaNet":
//     S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,   o_t = S_t q_t,
// evaluated chunk by chunk as in section "Three forms of one computation" (inside a chunk
// a masked C x C matrix, across chunks the carried state).  Per chunk of L <= 64 tokens,
// with the in-chunk log2-gate prefix lam_t, g_t = 2^lam_t, dec_t = 2^(lam_{L-1} - lam_t):
//
//   G  = [Q; K] K^T                                    (state independent)
//   A  = (Q K^T) * 2^(lam_t - lam_j), j <= t;   Lm = strictly-lower(diag(b) 2^(lam_t - lam_j) K K^T)
//   T  = (I + Lm)^-1;   W = T diag(b g) K;   U = T diag(b) V
//   P  = [diag(g) Q; W] S^T                            (state dependent: the chain)
//   E  = U - W S^T   (rows t: e_t = b_t (v_t - a_t S_{t-1} k_t), the delta-rule writes)
//   O  = diag(g) Q S^T + A E,   S^T <- g_{L-1} S^T + K^T diag(dec) E
//
// Rows of S evolve independently given the chunk's K, b and gates, so each head's d_v rows
// are split over kNS = 4 CTAs of 32 rows: the 32 heads of a B2 H16 workload give 128 CTAs,
// with no segments, transition pass or combine.  Every CTA forms the state-independent
// half itself (the four slices of a head run side by side and share its tiles through
// L2) one chunk ahead of the short state chain.  Roles:
//
//   warp 0       TMA producer: Q, K (two 64x64 boxes each) and the 64-column half of V
//                that holds the slice, into a ring of three stages; L2 prefetch ahead
//   warp 1       owns tensor memory
//   warp 3       gates: per stage the log2-gate prefix, beta, beta g and the column decay
//                factors, up to three chunks ahead (it completes the stage with the TMA)
//   warps 4-11   prep: A and Lm from G (masks, decays), the 64x64 inverse, T diag(b) and
//                T diag(b g); an elected thread issues G, W and U
//   warps 12-15  chain: [diag(g) Q; W] into tensor memory (the A operand of P), E from
//                U - W S^T, the state S^T (fp32, one d_k row of 32 values per thread) and
//                its bf16 copy, the outputs; elected threads issue P, dS and A E
//
// Each group issues its own products right after the named barrier that publishes their
// operands, so no product waits for a hand-off through another warp.  Product shapes
// (M x N x K, kind::f16, fp32 accumulators in tensor memory): G 128x64x128,
// W = [X; T diag(b g)] K 128x128x64 and U = [X; T diag(b)] V 128x64x64 (rows 64-127 are
// the result; X are the 64 rows of shared memory in front of the operand, whose products
// land in accumulator rows nobody reads), P 128x32x128 with A in tensor memory,
// dS^T = K^T E' 128x32x64 and A E 128x32x64 accumulated onto the rows 0-63 of P (again
// with 64 unused rows after the A tile).  Every wait is bounded; a timeout records an
// error, every role leaves its loop, in-flight copies and products are drained and the
// tensor memory is freed.
#include "la_internal.cuh"
#include "ptx.cuh"
#include "tc_util.cuh"
#include "tmap.cuh"
#include "bwd_util.cuh"

#include <cfloat>
#include <cstddef>
#include <cstring>

namespace la {
namespace {

using namespace ptx;
using namespace tc;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr int kNS = 4;           // d_v slices per head
constexpr int kDV = kD / kNS;    // 32 rows of S per CTA
constexpr int kStages = 3;
constexpr int kThreads = 512;
constexpr int kPrepT = 256;      // warps 4-11
constexpr int kChainT = 128;     // warps 12-15
// named barriers
constexpr uint32_t kBarPrep = 1, kBarChain = 3, kBarChainE = 4;
// A chunk whose column decay factor 2^(lam_{16b} - lam_j) inside a 16-token block exceeds
// 2^kFastSpan takes the exact per-element exponentials (no overflow in the fast factors).
constexpr float kFastSpan = 100.f;

// tensor memory columns
constexpr uint32_t kColG = 0;      // 64   G (fp32)
constexpr uint32_t kColW = 64;     // 128  W in lanes 64-127
constexpr uint32_t kColU = 192;    // 64   U (the V half) in lanes 64-127
constexpr uint32_t kColQW = 256;   // 2 x 64: [diag(g) Q; W] as bf16 pairs, per chunk parity
constexpr uint32_t kColP = 384;    // 2 x 32: P (+ A E) per chunk parity
constexpr uint32_t kColDS = 448;   // 32   dS^T
constexpr uint32_t kColU2 = 0;     // 64   two-pass variant: U of odd chunks (G is not formed)
constexpr uint32_t kTmemCols = 512;

// shared memory (bytes from the 1024-aligned base)
constexpr uint32_t kStage = 40960;                 // [Q0 | K0 | Q1 | K1 | V], 8 KB each
constexpr uint32_t kA0 = kStages * kStage;         // A tile, chunk parity 0 (8 KB)
constexpr uint32_t kA1 = kA0 + 8192;               // parity 1
constexpr uint32_t kTbg = kA1 + 8192;              // T diag(b g)   [t][j] bf16
constexpr uint32_t kTb = kTbg + 8192;              // T diag(b)
constexpr uint32_t kLm = kTb + 8192;               // fp32 64 x kTStride
constexpr uint32_t kTm = kLm + 64 * kTStride * 4;
constexpr uint32_t kZs = kTm + 64 * kTStride * 4;  // 4 x 272 floats
constexpr uint32_t kS = (kZs + 4 * 272 * 4 + 1023) & ~1023u;   // S^T bf16, 128 rows x 128 B
constexpr uint32_t kE = kS + 16384;                // E   [t] rows of 128 B (64 B used)
constexpr uint32_t kEp = kE + 8192;                // E' = diag(dec) E
constexpr uint32_t kSmall = kEp + 8192;

// Per-stage gate data, written by the gate warp: arrays read as float4 come first.
struct Gates {
    float lam[kC];   // inclusive prefix of log2(a) within the chunk
    float bet[kC];   // beta (0 past the end of the sequence)
    float bg[kC];    // beta 2^lam
    float cf[kC];    // 2^(lam_{16 floor(j/16)} - lam_j) >= 1
    int len;
    int slow;        // some cf exceeds 2^kFastSpan: exact exponentials for this chunk
    int pad[2];
};
struct Small {
    Gates gt[kStages];
    uint64_t full[kStages], empty[kStages];
    uint64_t g_done, wu_done, w_free, u_free;
    uint64_t p_done, ds_done;
    uint64_t ae_done[2];
    uint64_t a_full[2];   // two-pass variant: the A tile of each parity has arrived
    uint64_t u_free2[2];  // two-pass variant: U buffer of each parity read by the chain
    uint64_t qw_ready[2]; // two-pass variant: [diag(g) Q; W] of each parity in tensor memory
    uint64_t p_done2[2];  // two-pass variant: P of each parity done (its A operand is free)
    uint64_t p_issued;    // KDA variant: the chain has issued P of the next chunk
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Gates) % 16 == 0 && offsetof(Gates, cf) % 16 == 0, "float4 gate rows");
static_assert(kSmall % 16 == 0, "gate rows are read as float4");
constexpr uint32_t kBytes = kSmall + sizeof(Small);
static_assert(kBytes <= 227 * 1024, "shared memory per CTA");

// Shared-memory layouts of the variants (kSingle, kTwoGdn, kTwoKda).  The two-pass variant
// reads A, T diag(b) and T diag(b g) from pass 1: the stage carries the two T tiles after V
// (each 128-row A operand of W and U starts 8 KB before its tile, on the stage's own data),
// and the Lm, Tm and Zs buffers of the inverse are not needed.  The KDA variant's stage is
// [V | T diag(b) | K o 2^(lam_L - lam) | Gam_L]: Q o Gam and W go from pass 1's record
// straight into tensor memory, so no Q or K tile is staged.
constexpr int kSingle = 0, kTwoGdn = 1, kTwoKda = 2;
template <int VAR>
struct GLay;
template <>
struct GLay<kSingle> {
    static constexpr uint32_t kStage = ::la::kStage, kA0 = ::la::kA0, kA1 = ::la::kA1, kTbg = ::la::kTbg,
                              kTb = ::la::kTb, kLm = ::la::kLm, kTm = ::la::kTm, kZs = ::la::kZs,
                              kS = ::la::kS, kE = ::la::kE, kEp = ::la::kEp, kSmall = ::la::kSmall,
                              kBytes = ::la::kBytes;
    static constexpr uint32_t kVOff = 32768, kTbOff = 0, kTbgOff = 0, kKlOff = 8192, kKlHalf = 16384, kGlOff = 0;
};
template <>
struct GLay<kTwoGdn> {
    static constexpr uint32_t kStage = 57344;   // [Q0 | K0 | Q1 | K1 | V | T diag(b) | T diag(b g)]
    static constexpr uint32_t kVOff = 32768, kTbOff = 40960, kTbgOff = 49152, kKlOff = 8192, kKlHalf = 16384,
                              kGlOff = 0;
    static constexpr uint32_t kA0 = kStages * kStage, kA1 = kA0 + 8192;
    static constexpr uint32_t kTbg = 0, kTb = 0, kLm = 0, kTm = 0, kZs = 0;   // (not used)
    static constexpr uint32_t kS = kA1 + 8192, kE = kS + 16384, kEp = kE + 8192, kSmall = kEp + 8192;
    static constexpr uint32_t kBytes = kSmall + sizeof(Small);
};
template <>
struct GLay<kTwoKda> {
    static constexpr uint32_t kStage = 33792;   // [V | T diag(b) | K o 2^(lam_L - lam) (two halves) | Gam_L]
    static constexpr uint32_t kVOff = 0, kTbOff = 8192, kTbgOff = 0, kKlOff = 16384, kKlHalf = 8192,
                              kGlOff = 32768;
    static constexpr uint32_t kA0 = kStages * kStage, kA1 = kA0 + 8192;
    static constexpr uint32_t kTbg = 0, kTb = 0, kLm = 0, kTm = 0, kZs = 0;   // (not used)
    static constexpr uint32_t kS = kA1 + 8192, kE = kS + 16384, kEp = kE + 8192, kSmall = kEp + 8192;
    static constexpr uint32_t kBytes = kSmall + sizeof(Small);
};
static_assert(GLay<kTwoGdn>::kS % 1024 == 0 && GLay<kTwoGdn>::kA0 % 1024 == 0, "1024-byte aligned tiles");
static_assert(GLay<kTwoKda>::kS % 1024 == 0 && GLay<kTwoKda>::kA0 % 1024 == 0 && GLay<kTwoKda>::kStage % 1024 == 0,
              "1024-byte aligned tiles");
static_assert(GLay<kTwoGdn>::kBytes <= 227 * 1024 && GLay<kTwoKda>::kBytes <= 227 * 1024, "shared memory per CTA");

struct GdnParams {
    CUtensorMap tq, tk, tv;     // [BH][T][128] bf16, 64 x 64 boxes, 128B swizzle
    const float *gate;          // [BH][T] or nullptr (a = 1)
    const float *beta;          // [BH][T]
    __nv_bfloat16 *o;           // [BH][T][128]
    const float *s_in;          // nullable: zero start state
    float *s_out;
    long long seq_stride;       // state slot stride of a packed sequence (floats)
    const int *cu;              // packed sequences (nullptr: dense)
    int T, BH;
    unsigned *err;
    // two-pass variant: pass 1's per-chunk [A | T diag(b) | T diag(b g)] images,
    // [BH][nchunks][3][64 x 64] bf16 (nullptr: single pass)
    const __nv_bfloat16 *img;
    int nchunks;
};

__device__ __forceinline__ void gdn_range(const GdnParams &p, int unit, int &bh, int &seq, int &tb,
                                          int &te) {
    bh = unit % p.BH;
    seq = unit / p.BH;
    if (p.cu) {
        const int a = p.cu[seq], b = p.cu[seq + 1];
        tb = min(max(a, 0), p.T);
        te = min(max(b, tb), p.T);
        if ((a != tb || b != te) && threadIdx.x == 0 && p.err) atomicOr(p.err, (unsigned)kErrBadInput);
    } else {
        tb = 0;
        te = p.T;
    }
}

// One thread of a group polls `bar` (bounded wait); the group then meets at named barrier
// `id` of `n` threads, which also makes the decision to abandon uniform.  Waiting at the
// named barrier costs the other threads no issue slots.  False: abandon.
__device__ __forceinline__ bool group_wait(uint64_t *bar, uint32_t parity, bool poller, uint32_t id,
                                           uint32_t n, volatile int *abort, unsigned *err) {
    if (poller) mbar_wait(bar, parity, abort, err);
    return !named_sync_any(id, n, *abort != 0);
}

// D (+)= A B with A in tensor memory (K-major, 8 columns per K = 16 step) and B an
// MN-major shared-memory operand (rows of 128 bytes, 2048 bytes per step).
template <int NK>
__device__ __forceinline__ void mma_chain_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, bool accumulate_first) {
#pragma unroll
    for (int ks = 0; ks < NK; ++ks)
        mma_bf16_ts(d_tmem, a_tmem + 8 * ks, b_desc + (uint64_t)(ks * 128), idesc,
                    accumulate_first || ks > 0);
}

// 32 fp32 values as bf16 into the first 64 bytes (4 chunks) of row `row` of a 128B-swizzled
// MN-major tile.
__device__ __forceinline__ void st_row32_mn(uint32_t tile, uint32_t row, const float *v) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 w;
        w.x = pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]);
        w.y = pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]);
        w.z = pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]);
        w.w = pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]);
        sts128(tile + sw128_off(row, q), w);
    }
}

// ---------------------------------------------------------------------------------------
// Two-pass variant, pass 1: the state-independent factors of every chunk at once, two CTAs
// per SM over all (head row, chunk) pairs.  Per chunk it writes three bf16 64 x 64 tiles, each the 8 KB
// 128B-swizzled image the tensor cores read (rows of 128 bytes):
//   A = (Q K^T) 2^(lam_t - lam_j) (j <= t),   T diag(b),   T diag(b g)   (j <= t),
// T = (I + Lm)^-1, Lm = strictly-lower(diag(b) 2^(lam_t - lam_j) K K^T).  The Gram products
// run as warp-level tensor-core mma on the bf16 rows (m16n8k16, fp32 accumulate); every pair
// decay is one exponential (no factor outside [0, 1]).  The gate
// prefix is formed exactly as pass 2's gate warp forms it.
constexpr int kFacT = 256;
constexpr int kFacPitch = kD + 8;                              // bf16 pitch of the Q, K rows
constexpr uint32_t kFacTile = kC * kFacPitch * 2;              // 17408 B: a Q or K tile
static_assert(kFacTile == kC * kTStride * 4, "Lm / Tm reuse the Q / K tiles");
constexpr uint32_t kFacBuf = 2 * kFacTile;                     // [Q | K] of one chunk
constexpr uint32_t kFacZs = 2 * kFacBuf;                       // two chunk buffers, then Zs
constexpr uint32_t kFacImg = (kFacZs + 4 * 272 * 4 + 1023) & ~1023u;   // [A | T diag(b) | T diag(b g)]
constexpr uint32_t kFacG = kFacImg + 3 * 8192;                 // raw gate, beta [2][64] each
constexpr uint32_t kFacL = kFacG + 4 * kC * 4;                 // lam, bet, bg [64] each
constexpr uint32_t kFacBytes = kFacL + 3 * kC * 4;
constexpr int kImgHalves = 3 * 4096;                           // bf16 elements per chunk record

// Fused variant: q, k, v come from the token-major projections x through the short causal
// convolution (with the SiLU and the head-row L2 norm per flags) of the lesson page's
// section "Hybrids of 2025: Qwen3-Next and Kimi Linear", computed here as the rows arrive;
// the convolved q, k, v go out for pass 2 (and the caller).  The arithmetic is that of the
// stand-alone convolution kernel, operation for operation, so the two give the same bits.
struct FacConv {
    const __nv_bfloat16 *x[3];     // [B, T, H*128] token-major q, k, v projections
    const float *w[3];             // [H*128, width] taps
    const __nv_bfloat16 *win_in;   // [3, B, width-1, H*128] or nullptr (zeros)
    __nv_bfloat16 *win_out;        // [3, B, width-1, H*128] or nullptr (never overlaps win_in)
    __nv_bfloat16 *y;              // [3, B, H, T, 128] out
    int B, H, width;
    unsigned fqk, fv;              // LA_CONV_SILU | LA_CONV_L2NORM for q and k, for v
};
template <bool CONV>
struct FacLay {   // the raw rows of the fused variant carry the 3 tokens before the chunk
    static constexpr uint32_t kHalo = CONV ? 3 * kFacPitch * 2 : 0;
    static constexpr uint32_t kTile = kHalo + kFacTile;                   // one Q or K buffer
    static constexpr uint32_t kBuf = 2 * kTile;
    static constexpr uint32_t kZs = 2 * kBuf;
    static constexpr uint32_t kImg = (kZs + 4 * 272 * 4 + 1023) & ~1023u;  // also the raw v rows
    static constexpr uint32_t kG = kImg + 3 * 8192;
    static constexpr uint32_t kL = kG + 4 * kC * 4;
    static constexpr uint32_t kBytes = kL + 3 * kC * 4;
    static_assert(kHalo % 16 == 0 && kTile % 16 == 0, "16-byte rows");
    static_assert(67 * 256 <= 3 * 8192, "raw v rows fit the image area");
};
static_assert(FacLay<false>::kBytes == kFacBytes, "plain layout");

__device__ __forceinline__ float silu_tanh(float u) {   // u sigmoid(u), sigmoid = (1 + tanh(u/2)) / 2
    float t;
    const float h = 0.5f * u;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
    return fmaf(h, t, h);
}
__device__ __forceinline__ void unpack8(const uint4 &r, float (&f)[8]) {   // bf16 -> fp32 is exact
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        f[2 * j] = __uint_as_float(w[j] << 16);
        f[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
}
// Taps of 8 channels c0 .. c0 + 7 aligned to the window: e[3] multiplies the current token,
// e[k] (k < 3) the token 3 - k before it (zero where the width has no tap).
__device__ __forceinline__ void load_taps_aligned(const float *w, int width, size_t c0, float (&e)[4][8]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float *wc = w + (c0 + j) * width;
        e[3][j] = wc[width - 1];
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            const int i = k - (4 - width);   // tap index of the token 3 - k back
            e[k][j] = i >= 0 ? wc[i] : 0.f;
        }
    }
}
// One token's 8 channels: u = w[W-1] x_t + sum_{i < W-1} w[i] x_{t-(W-1)+i} (in that order),
// then SiLU and the head-row L2 norm per `fl` (the row's 16 chunks are the 16 lanes of a
// half-warp: every lane of the warp calls this together).  win[k] is the token 3 - k back.
__device__ __forceinline__ uint4 conv_token(const float (&e)[4][8], int width, const uint4 (&win)[3],
                                            const uint4 &xr, unsigned fl) {
    float x[8], u[8];
    unpack8(xr, x);
#pragma unroll
    for (int j = 0; j < 8; ++j) u[j] = e[3][j] * x[j];
#pragma unroll
    for (int k = 0; k < 3; ++k)
        if (k >= 4 - width) {
            float p[8];
            unpack8(win[k], p);
#pragma unroll
            for (int j = 0; j < 8; ++j) u[j] = fmaf(e[k][j], p[j], u[j]);
        }
    if (fl & LA_CONV_SILU)
#pragma unroll
        for (int j = 0; j < 8; ++j) u[j] = silu_tanh(u[j]);
    if (fl & LA_CONV_L2NORM) {
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) s = fmaf(u[j], u[j], s);
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        const float r = rsqrtf(s + 1e-6f);
#pragma unroll
        for (int j = 0; j < 8; ++j) u[j] *= r;
    }
    return make_uint4(pack_bf16x2(u[0], u[1]), pack_bf16x2(u[2], u[3]), pack_bf16x2(u[4], u[5]),
                      pack_bf16x2(u[6], u[7]));
}

// Each CTA takes chunks blockIdx.x, blockIdx.x + gridDim.x, ... (chunk i = head row i / nch,
// chunk i % nch); the next chunk's rows, gates and rates arrive by cp.async while the
// current one is processed.  Lm and Tm of the inverse take the places of the chunk's Q and
// K tiles once the Gram products have read them.  With CONV the staged rows are raw
// projections (3 tokens in front of the chunk included), convolved in place; the raw v
// rows arrive in the image area and are convolved straight out after the Gram products.
template <bool CONV>
__global__ void __launch_bounds__(kFacT, 2)
gdn_chunk_factors_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                         const float *__restrict__ gate, const float *__restrict__ beta, int T, int nch,
                         int total, __nv_bfloat16 *__restrict__ img, const FacConv cv) {
    using FL = FacLay<CONV>;
    extern __shared__ __align__(1024) uint8_t fsm[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float *Zs = reinterpret_cast<float *>(fsm + FL::kZs);
    uint8_t *im = fsm + FL::kImg;
    float *graw = reinterpret_cast<float *>(fsm + FL::kG), *braw = graw + 2 * kC;
    float *lam = reinterpret_cast<float *>(fsm + FL::kL), *bet = lam + kC, *bg = bet + kC;
    auto chunk_of = [&](int item, size_t &row0, int &L) {
        const int bh = item / nch, c = item % nch;
        row0 = (size_t)bh * T + (size_t)c * kC;
        L = min(kC, T - c * kC);
    };
    const int W1 = CONV ? cv.width - 1 : 0;
    const size_t Cx = CONV ? (size_t)cv.H * kD : 0;   // channels of a projection row
    // (fused) the 16-byte piece x8 .. x8 + 7 of head h's channels of projection z at token t
    // of batch row b: the projection, else the carried window, else nothing (zeros)
    auto raw_src = [&](int z, int b, int h, int t, int x8) -> const __nv_bfloat16 * {
        if (t >= T) return nullptr;
        // (selects, not an indexed parameter array: that would go through local memory)
        const __nv_bfloat16 *xz = z == 0 ? cv.x[0] : (z == 1 ? cv.x[1] : cv.x[2]);
        if (t >= 0) return xz + ((size_t)b * T + t) * Cx + (size_t)h * kD + x8;
        const int j = W1 + t;
        if (j < 0 || !cv.win_in) return nullptr;
        return cv.win_in + (((size_t)z * cv.B + b) * W1 + j) * Cx + (size_t)h * kD + x8;
    };
    // rows [0, L) of q and k (16-byte copies; rows past L zeroed), gates and rates
    auto stage = [&](int item, int buf) {
        size_t row0;
        int L;
        chunk_of(item, row0, L);
        uint8_t *base = fsm + buf * FL::kBuf;
        if constexpr (CONV) {   // 67 raw rows: tokens c*64 - 3 .. c*64 + 63
            const int bh = item / nch, c = item % nch, b = bh / cv.H, h = bh % cv.H;
            for (int p = tid; p < 2 * 67 * 16; p += kFacT) {
                const int which = p / (67 * 16), r = (p >> 4) % 67, x = p & 15;
                __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(base + which * FL::kTile) + r * kFacPitch + 8 * x;
                const __nv_bfloat16 *s = raw_src(which, b, h, c * kC - 3 + r, 8 * x);
                if (s) cp_async16(dst, s);
                else *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
            }
        } else {
            for (int p = tid; p < 2 * kC * 16; p += kFacT) {
                const int which = p >> 10, r = (p >> 4) & 63, x = p & 15;
                __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(base + which * FL::kTile) + r * kFacPitch + 8 * x;
                if (r < L) cp_async16(dst, (which ? k : q) + (row0 + r) * kD + 8 * x);
                else *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        if (tid < L) cp_async4(braw + buf * kC + tid, beta + row0 + tid);
        if (gate && tid >= 64 && tid - 64 < L) cp_async4(graw + buf * kC + tid - 64, gate + row0 + tid - 64);
        cp_async_commit();
    };
    if ((int)blockIdx.x < total) stage(blockIdx.x, 0);
    for (int item = blockIdx.x, it = 0; item < total; item += gridDim.x, ++it) {
        const int cur = it & 1;
        size_t row0;
        int L;
        chunk_of(item, row0, L);
        __nv_bfloat16 *Qs = reinterpret_cast<__nv_bfloat16 *>(fsm + cur * FL::kBuf + FL::kHalo);
        __nv_bfloat16 *Ks = reinterpret_cast<__nv_bfloat16 *>(fsm + cur * FL::kBuf + FL::kTile + FL::kHalo);
        float *Lm = reinterpret_cast<float *>(Qs);   // over Q
        float *Tm = reinterpret_cast<float *>(Ks);   // over K
        cp_async_wait_all();
        if (tid == 0) tma_store_wait_read<0>();   // the previous chunk's images have been read out
        __syncthreads();   // this chunk's rows are in; the other buffer and the images are free
        const bool pref = item + (int)gridDim.x < total;
        if constexpr (CONV) {
            const int bh = item / nch, c = item % nch, b = bh / cv.H, h = bh % cv.H;
            // the raw v rows into the image area (their own commit group, ahead of the prefetch)
            for (int p = tid; p < 67 * 16; p += kFacT) {
                const int r = p >> 4, x = p & 15;
                const __nv_bfloat16 *s = raw_src(2, b, h, c * kC - 3 + r, 8 * x);
                if (s) cp_async16(im + r * 256 + 16 * x, s);
                else *reinterpret_cast<uint4 *>(im + r * 256 + 16 * x) = make_uint4(0u, 0u, 0u, 0u);
            }
            cp_async_commit();
            if (c == nch - 1 && cv.win_out) {   // the carried windows after the sequence
                for (int p = tid; p < 3 * W1 * 16; p += kFacT) {
                    const int z = p / (W1 * 16), j = (p >> 4) % W1, x = p & 15;
                    const __nv_bfloat16 *s = raw_src(z, b, h, T - W1 + j, 8 * x);
                    *reinterpret_cast<uint4 *>(cv.win_out + (((size_t)z * cv.B + b) * W1 + j) * Cx + (size_t)h * kD + 8 * x) =
                        s ? *reinterpret_cast<const uint4 *>(s) : make_uint4(0u, 0u, 0u, 0u);
                }
            }
        }
        if (pref) stage(item + gridDim.x, cur ^ 1);
        if constexpr (CONV) {
            // q (threads 0-127) and k (128-255) in place: a thread takes the 8 channels cc of
            // tokens 8 rr .. 8 rr + 7, the 16 chunks of a token row in one half-warp
            const int z = tid >> 7, rr = (tid >> 4) & 7, cc = tid & 15;
            const int bh = item / nch, h = bh % cv.H;
            const uint32_t rows = smem_u32(fsm + cur * FL::kBuf + z * FL::kTile) + 16 * cc;
            float wr[4][8];
            load_taps_aligned(z ? cv.w[1] : cv.w[0], cv.width, (size_t)h * kD + 8 * cc, wr);
            // the 3 raw rows in front of the run are read before any thread replaces them
            uint4 win[3];
#pragma unroll
            for (int i = 0; i < 3; ++i) win[i] = lds128(rows + (8 * rr + i) * (kFacPitch * 2));
            __syncthreads();
#pragma unroll 2
            for (int i = 0; i < 8; ++i) {
                const int t = 8 * rr + i;
                const uint32_t a = rows + (t + 3) * (kFacPitch * 2);
                const uint4 xr = lds128(a);
                const uint4 o = conv_token(wr, cv.width, win, xr, cv.fqk);
                sts128(a, t < L ? o : make_uint4(0u, 0u, 0u, 0u));
                win[0] = win[1];
                win[1] = win[2];
                win[2] = xr;
            }
            fence_async_smem();   // the rows leave by bulk copies below
            __syncthreads();   // the chunk's q and k rows are convolved
            if (tid < 2 * kC && (tid & 63) < L) {   // row tid & 63 of q (threads 0-63) or k
                const int zz = tid >> 6, t = tid & 63;
                bulk_store(cv.y + (size_t)zz * cv.B * cv.H * T * kD + (row0 + t) * kD,
                           smem_u32(fsm + cur * FL::kBuf + zz * FL::kTile) + (t + 3) * (kFacPitch * 2), 2 * kD);
                tma_store_commit();
            }
        }
        if (warp == 0) {   // lane l takes tokens 2l, 2l + 1, as pass 2's gate warp
            float a0 = 1.f, a1 = 1.f, b0 = 0.f, b1 = 0.f;
            const int i0 = 2 * lane, i1 = 2 * lane + 1;
            if (i0 < L) {
                if (gate) a0 = graw[cur * kC + i0];
                b0 = braw[cur * kC + i0];
            }
            if (i1 < L) {
                if (gate) a1 = graw[cur * kC + i1];
                b1 = braw[cur * kC + i1];
            }
            const float g0 = (i0 < L) ? lg2(fmaxf(a0, FLT_MIN)) : 0.f;
            const float g1 = (i1 < L) ? lg2(fmaxf(a1, FLT_MIN)) : 0.f;
            float x = g0 + g1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float n = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += n;
            }
            const float l1 = x, l0 = x - g1;
            lam[i0] = l0;
            lam[i1] = l1;
            bet[i0] = b0;
            bet[i1] = b1;
            bg[i0] = b0 * ex2(l0);
            bg[i1] = b1 * ex2(l1);
        }
        // G = K K^T -> Lm (j < t), Q K^T -> A (j <= t): warp w rows 16 (w & 3), columns 32 (w >> 2)
        const int m0 = 16 * (warp & 3), n0 = 32 * (warp >> 2);
        const int g = lane >> 2, t4 = lane & 3;
        float gk[4][4] = {}, gq[4][4] = {};
#pragma unroll 4
        for (int kk = 0; kk < kD; kk += 16) {   // both products share the K fragments (ldmatrix)
            uint32_t ak[4], aq[4];
            frag_a<false>(ak, Ks, kFacPitch, m0, kk);
            frag_a<false>(aq, Qs, kFacPitch, m0, kk);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                uint32_t b[2];
                frag_b<false>(b, Ks, kFacPitch, kk, n0 + 8 * nt);
                mma_16x8x16_bf16(gk[nt], ak, b[0], b[1]);
                mma_16x8x16_bf16(gq[nt], aq, b[0], b[1]);
            }
        }
        if constexpr (CONV) {
            if (pref) asm volatile("cp.async.wait_group 1;" ::: "memory");   // the raw v rows
            else asm volatile("cp.async.wait_group 0;" ::: "memory");
            tma_store_wait_read<0>();   // the q, k rows have left the tiles
        }
        __syncthreads();   // Q and K read (Lm, Tm take their places); the gates are in
        if constexpr (CONV) {   // v: 16 runs of 4 tokens, straight out (no head norm unless asked)
            const int rr = tid >> 4, cc = tid & 15;
            const int bh = item / nch, h = bh % cv.H;
            const uint32_t rows = smem_u32(im) + 16 * cc;
            float wr[4][8];
            load_taps_aligned(cv.w[2], cv.width, (size_t)h * kD + 8 * cc, wr);
            uint4 win[3];
#pragma unroll
            for (int i = 0; i < 3; ++i) win[i] = lds128(rows + (4 * rr + i) * 256);
            __syncthreads();   // the rows in front of every run are read: convolve in place
#pragma unroll 2
            for (int i = 0; i < 4; ++i) {
                const int t = 4 * rr + i;
                const uint32_t a = rows + (t + 3) * 256;
                const uint4 xr = lds128(a);
                sts128(a, conv_token(wr, cv.width, win, xr, cv.fv));
                win[0] = win[1];
                win[1] = win[2];
                win[2] = xr;
            }
            fence_async_smem();
            __syncthreads();
            if (tid == 0) {   // the chunk's v rows are contiguous in shared and global memory
                bulk_store(cv.y + (size_t)2 * cv.B * cv.H * T * kD + row0 * kD, smem_u32(im) + 3 * 256, L * 2 * kD);
                tma_store_commit();
                tma_store_wait_read<0>();
            }
            __syncthreads();   // the v rows have left: the image area is free
        }
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int t = m0 + g + 8 * h, j = n0 + 8 * nt + 2 * t4;
                float a2[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int jj = j + e;
                    const float dd = jj <= t ? ex2(lam[t] - lam[jj]) : 0.f;
                    Lm[t * kTStride + jj] = jj < t ? bet[t] * gk[nt][2 * h + e] * dd : 0.f;
                    a2[e] = gq[nt][2 * h + e] * dd;
                }
                *reinterpret_cast<uint32_t *>(im + sw128_off(t, j >> 3) + (j & 7) * 2) = pack_bf16x2(a2[0], a2[1]);
            }
        __syncthreads();
        invert_unit_lower_rec<1, kFacT>(Lm, Tm, Zs, tid);
        __syncthreads();
        {   // T diag(b), T diag(b g) (lower triangle)
            const int t = tid >> 2, j0 = 16 * (tid & 3);
            float v1[16], v2[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const int j = j0 + jj;
                const float tj = (j <= t) ? Tm[t * kTStride + j] : 0.f;
                v1[jj] = tj * bet[j];
                v2[jj] = tj * bg[j];
            }
            st_row_bf16x16(smem_u32(im + 8192), t, j0 >> 3, v1);
            st_row_bf16x16(smem_u32(im + 16384), t, j0 >> 3, v2);
        }
        fence_async_smem();   // the images leave by a bulk copy
        __syncthreads();
        if (tid == 0) {
            bulk_store(img + (size_t)item * kImgHalves, smem_u32(im), 3 * 8192);
            tma_store_commit();
        }
    }
    cp_async_wait_all();
    tma_store_wait_all<0>();
}

// ---------------------------------------------------------------------------------------
// Kimi Delta Attention (mode 3: Diag(a_t) with one decay per channel c of d_k, section
// "The delta rule and Gated DeltaNet"), two-pass variant.  With the in-chunk log2 prefix
// lam_tc per channel, Gam_tc = 2^lam_tc and L the chunk's last token, the chunked form is
//   A_tj = sum_c q_tc k_jc 2^(lam_tc - lam_jc) (j <= t),
//   Lm_tj = b_t sum_c k_tc k_jc 2^(lam_tc - lam_jc) (j < t),   T = (I + Lm)^-1,
//   W = T diag(b) (K o Gam),   U = T diag(b) V,   E = U - W S^T,
//   O = (Q o Gam) S^T + A E,   S^T <- Diag(Gam_L) S^T + (K o 2^(lam_L - lam))^T E,
// so the chain of pass 2 is the gated-delta one with the decays moved into the operands.
// Pass 1 writes per chunk a record of bf16 128B-swizzled images (rows of 128 bytes):
constexpr uint32_t kKrA = 0;         // A                       64 x 64
constexpr uint32_t kKrTb = 8192;     // T diag(b)               64 x 64
constexpr uint32_t kKrQg = 16384;    // Q o Gam                 64 x 128 (two 64-column images)
constexpr uint32_t kKrW = 32768;     // W                       64 x 128
constexpr uint32_t kKrKl = 49152;    // K o 2^(lam_L - lam)     64 x 128
constexpr uint32_t kKrGl = 65536;    // Gam_L                   128 fp32
constexpr uint32_t kKdaRec = 66048;
// The Gram products A and Lm take the pair decay of 16-token blocks I (rows) and J <= I
// (columns) in three factors, with s_I the first token of block I and e_J the last of J:
//   2^(lam_t - lam_j) = 2^(lam_t - lam_{s_I})  [rows: F_t, in [2^-113, 1]]
//                     x 2^(lam_{s_I} - lam_{e_J}) [per channel, off the diagonal: D_IJ <= 1]
//                     x 2^(lam_{e_J} - lam_{s_J}) [per channel, off the diagonal: c_J <= 1]
//                     x 2^(lam_{s_J} - lam_j)  [columns: Fi_j, in [1, 2^113]].
// On a diagonal block (I = J) the middle factors are 1.  Off it, q_t F_t D_IJ <= 1 and
// k_j Fi_j c_J = k_j 2^(lam_{e_J} - lam_j) <= 1, so a factor that underflows belongs to a
// pair weight below 2^-126.  F and Fi span at most 15 tokens of decay, which stays inside
// the exponent range because the Gram products bound each log2 gate below at
// kGramLog2Floor (a >= 0.0055): only pair weights across such a gate, already below 0.0055,
// move.  Every state-facing factor (Gam, 2^(lam_L - lam), Gam_L) takes the gates exactly.
constexpr float kGramLog2Floor = -7.5f;
constexpr int kKP = kD + 8;                               // bf16 pitch of the Q, K, K-hat, K o Gam rows
constexpr uint32_t kKT = kC * kKP * 2;                    // 17408 B
static_assert(kKT == kC * kTStride * 4, "Lm / Tm take the places of the Q / K rows");
constexpr uint32_t kkQ = 0;                               // Q rows, scaled by F in place; then Lm
constexpr uint32_t kkK = kkQ + kKT;                       // K rows, scaled by F in place; then Tm; then W
constexpr uint32_t kkR = kkK + kKT;                       // raw gates [64][128]; then the Q o Gam, K o 2^(lam_L - lam) images
constexpr uint32_t kkH = kkR + kC * kD * 4;               // K-hat = K o Fi; then the A, T diag(b) images
constexpr uint32_t kkG = kkH + kKT;                       // K o Gam (the B operand of W)
constexpr uint32_t kkZ = kkG + kKT;                       // Zs of the inverse
constexpr uint32_t kkS = kkZ + 4 * 272 * 4;               // per 16-token block and channel pair: sums, first steps
constexpr uint32_t kkB = kkS + 4 * 64 * 16 + 4 * 64 * 8;  // beta [64]
constexpr uint32_t kkF = kkB + kC * 4;                    // D_IJ [6][64], c_J [3][64] bf16 pairs
constexpr uint32_t kkBytes = kkF + 9 * 64 * 4;
static_assert(2 * (kkBytes + 1024) <= 228 * 1024, "two CTAs per SM");

// byte offset of element (t, c) in a pair of 64-column 128B-swizzled images
__device__ __forceinline__ uint32_t img2_off(int t, int c) {
    return (uint32_t)(c >> 6) * 8192u + sw128_off(t, (c & 63) >> 3) + (uint32_t)(c & 7) * 2u;
}
__device__ __forceinline__ uint32_t hmul_bf16x2(uint32_t a, uint32_t b) {
    const __nv_bfloat162 r = __hmul2(*reinterpret_cast<const __nv_bfloat162 *>(&a),
                                     *reinterpret_cast<const __nv_bfloat162 *>(&b));
    return *reinterpret_cast<const uint32_t *>(&r);
}

// Two CTAs per SM over all (head row, chunk) pairs, one chunk at a time; the next chunk's
// rows are prefetched into L2 while the current one is processed.
__global__ void __launch_bounds__(kFacT, 2)
kda_chunk_factors_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                         const float *__restrict__ gate, const float *__restrict__ beta, int T, int nch,
                         int total, uint8_t *__restrict__ rec) {
    extern __shared__ __align__(1024) uint8_t ksm[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    __nv_bfloat16 *Qs = reinterpret_cast<__nv_bfloat16 *>(ksm + kkQ);
    __nv_bfloat16 *Ks = reinterpret_cast<__nv_bfloat16 *>(ksm + kkK);
    __nv_bfloat16 *Kh = reinterpret_cast<__nv_bfloat16 *>(ksm + kkH);
    __nv_bfloat16 *Kg = reinterpret_cast<__nv_bfloat16 *>(ksm + kkG);
    float *Gr = reinterpret_cast<float *>(ksm + kkR);
    float *Lm = reinterpret_cast<float *>(ksm + kkQ), *Tm = reinterpret_cast<float *>(ksm + kkK);
    float *Zs = reinterpret_cast<float *>(ksm + kkZ), *bet = reinterpret_cast<float *>(ksm + kkB);
    float4 *bsum = reinterpret_cast<float4 *>(ksm + kkS);      // [block][pair]: exact sums (2), bounded sums (2)
    float2 *bfirst = reinterpret_cast<float2 *>(ksm + kkS + 4 * 64 * 16);   // [block][pair]: bounded first steps
    const uint32_t *Dp = reinterpret_cast<const uint32_t *>(ksm + kkF);   // [9][64] bf16 pairs
    uint8_t *imR = ksm + kkR, *imA = ksm + kkH, *imW = ksm + kkK;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        const int c0 = item % nch;
        const size_t row0 = (size_t)(item / nch) * T + (size_t)c0 * kC;
        const int L = min(kC, T - c0 * kC);
        uint8_t *rc = rec + (size_t)item * kKdaRec;
        // ---- rows [0, L) of q, k and the gates (rows past L: zero; their gates are not read), beta
        for (int p = tid; p < 2 * kC * 16; p += kFacT) {
            const int which = p >> 10, r = (p >> 4) & 63, x = p & 15;
            __nv_bfloat16 *dst = (which ? Ks : Qs) + r * kKP + 8 * x;
            if (r < L) cp_async16(dst, (which ? k : q) + (row0 + r) * kD + 8 * x);
            else *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
        }
        if (gate)
            for (int p = tid; p < L * 32; p += kFacT) cp_async16(Gr + 4 * p, gate + row0 * kD + 4 * p);
        cp_async_commit();
        if (tid < kC) bet[tid] = tid < L ? beta[row0 + tid] : 0.f;
        cp_async_wait_all();
        __syncthreads();
        // ---- thread (channel pair cp, 16-token block J0): the prefixes of channels 2 cp, 2 cp + 1
        // inside the block, exact (lx) and with the Gram products' bound (lb)
        const int cp = tid & 63, J0 = tid >> 6, c2 = 2 * cp;
        float lx[16][2], lb[16][2];
        {
            float sx0 = 0.f, sx1 = 0.f, sb0 = 0.f, sb1 = 0.f, f0 = 0.f, f1 = 0.f;
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const int t = 16 * J0 + m;
                float g0 = 0.f, g1 = 0.f;
                if (gate && t < L) {
                    const float2 a = *reinterpret_cast<const float2 *>(Gr + t * kD + c2);
                    g0 = lg2(fmaxf(a.x, FLT_MIN));
                    g1 = lg2(fmaxf(a.y, FLT_MIN));
                }
                const float h0 = fmaxf(g0, kGramLog2Floor), h1 = fmaxf(g1, kGramLog2Floor);
                if (m == 0) {
                    f0 = h0;
                    f1 = h1;
                }
                sx0 += g0;
                sx1 += g1;
                sb0 += h0;
                sb1 += h1;
                lx[m][0] = sx0;
                lx[m][1] = sx1;
                lb[m][0] = sb0;
                lb[m][1] = sb1;
            }
            bsum[J0 * 64 + cp] = make_float4(sx0, sx1, sb0, sb1);
            bfirst[J0 * 64 + cp] = make_float2(f0, f1);
        }
        __syncthreads();   // the block sums are in; the raw gates are read
        // exact prefix before the block and at the chunk's last token
        float ox0 = 0.f, ox1 = 0.f, lL0 = 0.f, lL1 = 0.f;
#pragma unroll
        for (int J = 0; J < 4; ++J) {
            const float4 v = bsum[J * 64 + cp];
            if (J < J0) {
                ox0 += v.x;
                ox1 += v.y;
            }
            lL0 += v.x;
            lL1 += v.y;
        }
        if (J0 == 0) *reinterpret_cast<float2 *>(rc + kKrGl + 4 * c2) = make_float2(ex2(lL0), ex2(lL1));
        if (tid < 64) {    // D_IJ = 2^(lam_{s_I} - lam_{e_J}) (I > J), c_J = 2^(lam_{e_J} - lam_{s_J}) (J < 3)
            float tb[4][2], fb[4][2];
#pragma unroll
            for (int J = 0; J < 4; ++J) {
                const float4 v = bsum[J * 64 + cp];
                const float2 f = bfirst[J * 64 + cp];
                tb[J][0] = v.z;
                tb[J][1] = v.w;
                fb[J][0] = f.x;
                fb[J][1] = f.y;
            }
            auto pair = [&](float a0, float a1) {
                const __nv_bfloat162 h = __floats2bfloat162_rn(ex2(a0), ex2(a1));
                return *reinterpret_cast<const uint32_t *>(&h);
            };
            uint32_t *D = reinterpret_cast<uint32_t *>(ksm + kkF);
#pragma unroll
            for (int I = 1; I < 4; ++I)
#pragma unroll
                for (int J = 0; J < I; ++J) {   // lam_{s_I} - lam_{e_J}: I's first step and the blocks between
                    float e0 = fb[I][0], e1 = fb[I][1];
#pragma unroll
                    for (int K = J + 1; K < I; ++K) {
                        e0 += tb[K][0];
                        e1 += tb[K][1];
                    }
                    D[(I * (I - 1) / 2 + J) * 64 + cp] = pair(e0, e1);
                }
#pragma unroll
            for (int J = 0; J < 3; ++J) D[(6 + J) * 64 + cp] = pair(tb[J][0] - fb[J][0], tb[J][1] - fb[J][1]);
        }
        // ---- per element pair: Q o Gam and K o 2^(lam_L - lam) (images, for the record), K o Gam
        // (for W), and the Gram operands Q F, K F (in place) and K Fi, F = 2^(lb - lb_{s_J0})
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const int t = 16 * J0 + m;
            const float2 qv = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(Qs + t * kKP + c2));
            const float2 kv = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(Ks + t * kKP + c2));
            const float l0 = lx[m][0] + ox0, l1 = lx[m][1] + ox1;
            const float gm0 = ex2(l0), gm1 = ex2(l1);
            const float d0 = lb[m][0] - lb[0][0], d1 = lb[m][1] - lb[0][1];   // <= 0, >= 15 kGramLog2Floor
            const float fa0 = ex2(d0), fa1 = ex2(d1);
            const float fi0 = ex2(-d0), fi1 = ex2(-d1);
            const uint32_t o = img2_off(t, c2);
            *reinterpret_cast<uint32_t *>(imR + o) = pack_bf16x2(qv.x * gm0, qv.y * gm1);
            *reinterpret_cast<uint32_t *>(imR + 16384 + o) =
                pack_bf16x2(kv.x * ex2(lL0 - l0), kv.y * ex2(lL1 - l1));
            *reinterpret_cast<uint32_t *>(Kg + t * kKP + c2) = pack_bf16x2(kv.x * gm0, kv.y * gm1);
            *reinterpret_cast<uint32_t *>(Qs + t * kKP + c2) = pack_bf16x2(qv.x * fa0, qv.y * fa1);
            *reinterpret_cast<uint32_t *>(Ks + t * kKP + c2) = pack_bf16x2(kv.x * fa0, kv.y * fa1);
            *reinterpret_cast<uint32_t *>(Kh + t * kKP + c2) = pack_bf16x2(kv.x * fi0, kv.y * fi1);
        }
        __syncthreads();   // the operands and the block factors are in
        // ---- Gram products: warp w rows 16 (w & 3) (block I), columns 32 (w >> 2) (blocks J)
        const int I = warp & 3, Jp = warp >> 2, m0 = 16 * I;
        const int g = lane >> 2, t4 = lane & 3;
        float gq[2][2][4] = {}, gk[2][2][4] = {};
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            const int J = 2 * Jp + jj;
            if (J > I) continue;   // (warp-uniform)
            const uint32_t *DI = Dp + (I * (I - 1) / 2 + J) * 64, *CJ = Dp + (6 + J) * 64;
#pragma unroll 4
            for (int kk = 0; kk < kD; kk += 16) {
                uint32_t aq[4], ak[4];
                frag_a<false>(aq, Qs, kKP, m0, kk);
                frag_a<false>(ak, Ks, kKP, m0, kk);
                uint32_t dd[2] = {0u, 0u}, cc[2] = {0u, 0u};
                if (J < I) {   // fragment registers i hold channel pairs kk/2 + t4 + 4 (i >> 1)
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        dd[i] = DI[kk / 2 + t4 + 4 * i];
                        cc[i] = CJ[kk / 2 + t4 + 4 * i];
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        aq[i] = hmul_bf16x2(aq[i], dd[i >> 1]);
                        ak[i] = hmul_bf16x2(ak[i], dd[i >> 1]);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    uint32_t b[2];
                    frag_b<false>(b, Kh, kKP, kk, 16 * J + 8 * nt);
                    if (J < I) {
                        b[0] = hmul_bf16x2(b[0], cc[0]);
                        b[1] = hmul_bf16x2(b[1], cc[1]);
                    }
                    mma_16x8x16_bf16(gq[jj][nt], aq, b[0], b[1]);
                    mma_16x8x16_bf16(gk[jj][nt], ak, b[0], b[1]);
                }
            }
        }
        // the next chunk's rows into L2
        if (item + (int)gridDim.x < total) {
            const int nx = item + gridDim.x, nc = nx % nch;
            const size_t nrow = (size_t)(nx / nch) * T + (size_t)nc * kC;
            const int nL = min(kC, T - nc * kC);
            for (int p = tid; p < 8 * kC; p += kFacT) {   // per row: 2 lines of q, 2 of k, 4 of gates
                const int r = p >> 3, z = p & 7;
                if (r >= nL) continue;
                if (z < 2) prefetch_l2(q + (nrow + r) * kD + 64 * z);
                else if (z < 4) prefetch_l2(k + (nrow + r) * kD + 64 * (z - 2));
                else if (gate) prefetch_l2(gate + (nrow + r) * kD + 32 * (z - 4));
            }
        }
        __syncthreads();   // the operands are read: Lm over Q, the A image over K-hat
#pragma unroll
        for (int jj = 0; jj < 2; ++jj)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int t = m0 + g + 8 * h, j = 32 * Jp + 16 * jj + 8 * nt + 2 * t4;
                    float a2[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int je = j + e;
                        Lm[t * kTStride + je] = je < t ? bet[t] * gk[jj][nt][2 * h + e] : 0.f;
                        a2[e] = je <= t ? gq[jj][nt][2 * h + e] : 0.f;
                    }
                    *reinterpret_cast<uint32_t *>(imA + sw128_off(t, j >> 3) + (j & 7) * 2) = pack_bf16x2(a2[0], a2[1]);
                }
        __syncthreads();
        invert_unit_lower_rec<1, kFacT>(Lm, Tm, Zs, tid);
        __syncthreads();
        {   // T diag(b) (lower triangle)
            const int t = tid >> 2, j0 = 16 * (tid & 3);
            float v1[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const int j = j0 + jj;
                v1[jj] = (j <= t) ? Tm[t * kTStride + j] * bet[j] : 0.f;
            }
            st_row_bf16x16(smem_u32(imA + 8192), t, j0 >> 3, v1);
        }
        __syncthreads();
        {   // W = T diag(b) (K o Gam): warp w rows 16 (w & 3), channels 64 (w >> 2); images over Tm
            const int n0 = 64 * Jp;
            const __nv_bfloat16 *Tb = reinterpret_cast<const __nv_bfloat16 *>(imA + 8192);
            float acc[8][4] = {};
#pragma unroll
            for (int kk = 0; kk < kC; kk += 16) {
                uint32_t a[4];
                frag_a_sw64(a, Tb, m0, kk);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    uint32_t b[2];
                    frag_b<true>(b, Kg, kKP, kk, n0 + 8 * nt);
                    mma_16x8x16_bf16(acc[nt], a, b[0], b[1]);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int t = m0 + g + 8 * h, c = n0 + 8 * nt + 2 * t4;
                    *reinterpret_cast<uint32_t *>(imW + img2_off(t, c)) = pack_bf16x2(acc[nt][2 * h], acc[nt][2 * h + 1]);
                }
        }
        __syncthreads();
        fence_async_smem();   // the images leave by bulk copies
        __syncthreads();
        if (tid == 0) {   // the record: A and T diag(b), Q o Gam, W, K o 2^(lam_L - lam)
            bulk_store(rc + kKrA, smem_u32(imA), 16384);
            bulk_store(rc + kKrQg, smem_u32(imR), 16384);
            bulk_store(rc + kKrW, smem_u32(imW), 16384);
            bulk_store(rc + kKrKl, smem_u32(imR + 16384), 16384);
            tma_store_commit();
            tma_store_wait_read<0>();   // (before the next chunk's rows land on the images)
        }
        __syncthreads();
    }
    if (tid == 0) tma_store_wait_all<0>();
}

template <int VAR>
__global__ void __launch_bounds__(kThreads, 1) gdn_prefill_kernel(const __grid_constant__ GdnParams p) {
    constexpr bool TWO = VAR != kSingle, KDA = VAR == kTwoKda;
    using GL = GLay<VAR>;
    // pass 1's record of chunk c of this head row (two-pass variants)
    auto record = [&](int bh_, int c_) -> const uint8_t * {
        return reinterpret_cast<const uint8_t *>(p.img) +
               ((size_t)bh_ * p.nchunks + c_) * (size_t)(KDA ? kKdaRec : 2 * kImgHalves);
    };
    // the variant's layout (shadows the single-pass constants)
    constexpr uint32_t kStage = GL::kStage, kA0 = GL::kA0, kA1 = GL::kA1, kTbg = GL::kTbg, kTb = GL::kTb,
                       kLm = GL::kLm, kTm = GL::kTm, kZs = GL::kZs, kS = GL::kS, kE = GL::kE, kEp = GL::kEp,
                       kSmall = GL::kSmall;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sb = smem_u32(smem_raw);
    if (sb & 1023u) {
        if (threadIdx.x == 0 && p.err) atomicOr(p.err, (unsigned)kErrBadLaunch);
        return;
    }
    Small *sm = reinterpret_cast<Small *>(smem_raw + kSmall);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int vs = blockIdx.x % kNS;           // d_v slice: rows [32 vs, 32 vs + 32) of S
    int bh, seq, tb, te;
    gdn_range(p, blockIdx.x / kNS, bh, seq, tb, te);
    if (te <= tb) return;   // an empty packed sequence
    const int nch = (te - tb + kC - 1) / kC;
    const size_t slot = (size_t)seq * p.seq_stride + (size_t)bh * kD * kD;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm->full[s], 2);   // the TMA bytes and the gate warp
            mbar_init(&sm->empty[s], 1);
        }
        mbar_init(&sm->g_done, 1);
        mbar_init(&sm->wu_done, 1);
        mbar_init(&sm->w_free, 1);
        mbar_init(&sm->u_free, 1);
        mbar_init(&sm->p_done, 1);
        mbar_init(&sm->ds_done, 1);
        mbar_init(&sm->ae_done[0], 1);
        mbar_init(&sm->ae_done[1], 1);
        mbar_init(&sm->a_full[0], 1);
        mbar_init(&sm->a_full[1], 1);
        mbar_init(&sm->u_free2[0], 1);
        mbar_init(&sm->u_free2[1], 1);
        mbar_init(&sm->qw_ready[0], 1);
        mbar_init(&sm->qw_ready[1], 1);
        mbar_init(&sm->p_done2[0], 1);
        mbar_init(&sm->p_done2[1], 1);
        mbar_init(&sm->p_issued, 1);
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
    // instruction descriptors
    const uint32_t id_g = idesc_bf16(128, 64, false, false);
    const uint32_t id_w = idesc_bf16(128, 128, false, true);
    const uint32_t id_u = idesc_bf16(128, 64, false, true);
    const uint32_t id_p = idesc_bf16(128, kDV, false, true);
    const uint32_t id_ds = idesc_bf16(128, kDV, true, true);
    const uint32_t id_ae = idesc_bf16(128, kDV, false, true);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            if (!KDA) {
                tma_prefetch_desc(&p.tq);
                tma_prefetch_desc(&p.tk);
            }
            tma_prefetch_desc(&p.tv);
            const int vx = 64 * (vs >> 1);
            int issued[kStages] = {0, 0, 0};
            for (int c = 0; c < nch; ++c) {
                const int s = c % kStages, u = c / kStages;
                if (u >= 1 && !mbar_wait(&sm->empty[s], (u - 1) & 1, abort, p.err)) break;
                const uint32_t st = sb + s * kStage;
                const int t = tb + kC * c;
                if constexpr (KDA) {   // V, then T diag(b), K o 2^(lam_L - lam) and Gam_L (pass 1)
                    const uint8_t *rec = record(bh, c);
                    mbar_arrive_expect_tx(&sm->full[s], 8192 + 8192 + 16384 + 512);
                    tma_load_3d(st + GL::kVOff, &p.tv, vx, t, bh, &sm->full[s]);
                    bulk_load(st + GL::kTbOff, rec + kKrTb, 8192, &sm->full[s]);
                    bulk_load(st + GL::kKlOff, rec + kKrKl, 16384, &sm->full[s]);
                    bulk_load(st + GL::kGlOff, rec + kKrGl, 512, &sm->full[s]);
                } else {
                    mbar_arrive_expect_tx(&sm->full[s], kStage);
                    tma_load_3d(st + 0, &p.tq, 0, t, bh, &sm->full[s]);
                    tma_load_3d(st + 8192, &p.tk, 0, t, bh, &sm->full[s]);
                    tma_load_3d(st + 16384, &p.tq, 64, t, bh, &sm->full[s]);
                    tma_load_3d(st + 24576, &p.tk, 64, t, bh, &sm->full[s]);
                    tma_load_3d(st + 32768, &p.tv, vx, t, bh, &sm->full[s]);
                    if constexpr (TWO) {   // T diag(b), T diag(b g) of chunk c (pass 1)
                        const uint8_t *rec = record(bh, c);
                        bulk_load(st + GL::kTbOff, rec + 8192, 8192, &sm->full[s]);
                        bulk_load(st + GL::kTbgOff, rec + 16384, 8192, &sm->full[s]);
                    }
                }
                issued[s] = u + 1;
                // the chunk three ahead of this one into L2 (the slices of a head share it)
                const int tp = t + kStages * kC;
                if (tp < te) {
                    if constexpr (KDA) {
                        bulk_prefetch_l2(record(bh, c + kStages), kKdaRec);
                    } else {
                        tma_prefetch_l2_3d(&p.tq, 0, tp, bh);
                        tma_prefetch_l2_3d(&p.tq, 64, tp, bh);
                        tma_prefetch_l2_3d(&p.tk, 0, tp, bh);
                        tma_prefetch_l2_3d(&p.tk, 64, tp, bh);
                    }
                    tma_prefetch_l2_3d(&p.tv, vx, tp, bh);
                }
            }
            for (int s = 0; s < kStages; ++s)
                if (issued[s] > 0) drain_wait(&sm->full[s], (issued[s] - 1) & 1);
        }
    } else if (warp == 3) {
        // ------------------------------------------------------------ gates
        // lane l takes tokens 2l, 2l + 1 of the chunk
        for (int c = 0; c < nch; ++c) {
            const int s = c % kStages, u = c / kStages;
            if (u >= 1 && !mbar_wait(&sm->empty[s], (u - 1) & 1, abort, p.err)) break;
            const int t0 = tb + kC * c;
            const int L = min(kC, te - t0);
            float a0 = 1.f, a1 = 1.f, b0 = 0.f, b1 = 0.f;
            const int i0 = 2 * lane, i1 = 2 * lane + 1;
            const size_t base = (size_t)bh * p.T + t0;
            if (i0 < L) {
                if (p.gate) a0 = p.gate[base + i0];
                b0 = p.beta[base + i0];
            }
            if (i1 < L) {
                if (p.gate) a1 = p.gate[base + i1];
                b1 = p.beta[base + i1];
            }
            const float g0 = (i0 < L) ? lg2(fmaxf(a0, FLT_MIN)) : 0.f;
            const float g1 = (i1 < L) ? lg2(fmaxf(a1, FLT_MIN)) : 0.f;
            float x = g0 + g1;   // inclusive scan of the pair sums over the lanes
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float n = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += n;
            }
            const float l1 = x, l0 = x - g1;    // prefixes at tokens 2l + 1 and 2l
            // lam at the first token of the 16-token block (lane 8 floor(l / 8), token 0)
            const float lb = __shfl_sync(0xffffffffu, l0, lane & ~7);
            Gates *G = &sm->gt[s];
            reinterpret_cast<float2 *>(G->lam)[lane] = make_float2(l0, l1);
            reinterpret_cast<float2 *>(G->bet)[lane] = make_float2(b0, b1);
            reinterpret_cast<float2 *>(G->bg)[lane] = make_float2(b0 * ex2(l0), b1 * ex2(l1));
            reinterpret_cast<float2 *>(G->cf)[lane] = make_float2(ex2(lb - l0), ex2(lb - l1));
            const bool slow = __any_sync(0xffffffffu, lb - l1 > kFastSpan);
            if (lane == 0) {
                G->len = L;
                G->slow = slow ? 1 : 0;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->full[s]);
        }
    } else if (warp >= 4 && warp < 12) {
        // ------------------------------------------------------------ prep warps 4-11
        if constexpr (TWO) {
            // Two-pass: thread 128 copies each chunk's A tile and issues W and U from the
            // stage's T tiles (the factors themselves came from pass 1); the eight warps then
            // write [diag(g) Q; W] of the chunk into tensor memory as the A operand of P, a
            // chunk or two ahead of the chain, which only waits for it (qw_ready).
            const int pq = warp & 3, ph = (warp - 4) >> 2;   // lane quarter; which half of the work
            const uint32_t tl = tm + ((uint32_t)(32 * pq) << 16);
            const int prow = 32 * pq + lane;
            const bool lead = threadIdx.x == 128;
            int issued[2] = {0, 0};
            for (int c = 0; c < nch; ++c) {
                const int s = c % kStages, b = c & 1;
                bool ok = true;
                // KDA: this thread's half row of Q o Gam (rows 0-63) or W (rows 64-127), read
                // from the record before the waits below
                uint4 pre[8];
                if constexpr (KDA) {
                    const uint8_t *src = record(bh, c) + (pq < 2 ? kKrQg : kKrW) + 8192 * ph;
                    const int t = prow & 63;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) pre[ch] = *reinterpret_cast<const uint4 *>(src + sw128_off(t, ch));
                }
                if (lead) {
                    // A(c) into its parity buffer once A E(c - 2) has read it
                    ok = c < 2 || mbar_wait(&sm->ae_done[b], ((c >> 1) - 1) & 1, abort, p.err);
                    if (ok) {
                        mbar_arrive_expect_tx(&sm->a_full[b], 8192);
                        bulk_load(sb + (b ? kA1 : kA0), record(bh, c), 8192, &sm->a_full[b]);
                        issued[b] = (c >> 1) + 1;
                    }
                    // W = T diag(b g) K, U = T diag(b) V (rows 64-127) once the stage is in, W(c - 1)
                    // was read (the group's own step below) and U(c - 2) was read by the chain
                    // (U has a buffer per chunk parity)
                    // ... and (KDA: U alone, W comes from pass 1), so that it queues behind the
                    // chain's P(c - 1) instead of in front of it (the tensor pipe runs in issue
                    // order), once P(c - 1) has been issued: it then runs while the chain forms
                    // E(c - 1).  (The gated delta rule issues W and U as early as it can: W(c)
                    // has to be converted into the operand of P(c) in time.)
                    ok = ok && mbar_wait(&sm->full[s], (c / kStages) & 1, abort, p.err) &&
                         (c < 2 || mbar_wait(&sm->u_free2[b], ((c >> 1) - 1) & 1, abort, p.err)) &&
                         (!KDA || c < 1 || mbar_wait(&sm->p_issued, (c - 1) & 1, abort, p.err));
                    if (ok) {
                        tc_fence_after();
                        const uint32_t st = sb + s * kStage;
                        if (!KDA)   // (KDA: W comes from pass 1)
                            mma_chain<4, true, false>(tm + kColW, dk(st + GL::kTbgOff - 8192),
                                                      dmn(st + 8192, 16384), id_w, false);
                        mma_chain<4, true, false>(tm + (b ? kColU2 : kColU), dk(st + GL::kTbOff - 8192),
                                                  dmn(st + GL::kVOff, 8192), id_u, false);
                        mma_commit(&sm->wu_done);
                        // W(c) formed, and P(c - 2) done with this parity's A operand buffer
                        ok = mbar_wait(&sm->wu_done, c & 1, abort, p.err) &&
                             (c < 2 || mbar_wait(&sm->p_done2[b], ((c >> 1) - 1) & 1, abort, p.err));
                    }
                }
                // every thread reads the stage's Q tile and gates
                mbar_wait(&sm->full[s], (c / kStages) & 1, abort, p.err);
                if (named_sync_any(kBarPrep, kPrepT, !ok || *abort != 0)) break;
                tc_fence_after();
                const uint32_t dst = tl + kColQW + 64 * b;
                if constexpr (KDA) {   // rows 0-63: Q o Gam, rows 64-127: W, column half ph
                    uint32_t w[32];
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        w[4 * ch + 0] = pre[ch].x;
                        w[4 * ch + 1] = pre[ch].y;
                        w[4 * ch + 2] = pre[ch].z;
                        w[4 * ch + 3] = pre[ch].w;
                    }
                    tmem_st32(dst + 32 * ph, w);
                } else if (pq < 2) {   // rows 0-63: diag(g) Q, column half ph
                    const int t = prow;
                    const float gt = ex2(sm->gt[s].lam[t]);
                    const uint32_t st = sb + s * kStage;
                    uint32_t w[32];
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        const uint4 x = scale_bf16x8(lds128(st + 16384 * ph + sw128_off(t, ch)), gt);
                        w[4 * ch + 0] = x.x;
                        w[4 * ch + 1] = x.y;
                        w[4 * ch + 2] = x.z;
                        w[4 * ch + 3] = x.w;
                    }
                    tmem_st32(dst + 32 * ph, w);
                } else {        // rows 64-127: W as bf16, column quarters 2 ph, 2 ph + 1
#pragma unroll 1
                    for (int hh = 0; hh < 2; ++hh) {
                        const int h = 2 * ph + hh;
                        float f[32];
                        tmem_ld32(tl + kColW + 32 * h, f);
                        uint32_t w[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(f[2 * j], f[2 * j + 1]);
                        tmem_st16u(dst + 16 * h, w);
                    }
                }
                tc_fence_before();
                named_sync(kBarPrep, kPrepT);
                if (lead) {
                    mbar_arrive(&sm->w_free);
                    // A(c) has arrived too: the chain's A E(c) needs no wait of its own
                    if (!mbar_wait(&sm->a_full[b], (c >> 1) & 1, abort, p.err)) break;
                    mbar_arrive(&sm->qw_ready[b]);
                }
            }
            if (lead) {   // nothing issued here may still write tensor or shared memory at exit
                mma_commit(&sm->g_done);
                drain_wait(&sm->g_done, 0);
                for (int bb = 0; bb < 2; ++bb)
                    if (issued[bb] > 0) drain_wait(&sm->a_full[bb], (issued[bb] - 1) & 1);
            }
        } else {
        const int pe = threadIdx.x - 128;           // 0..255
        const int pq = warp & 3;                    // tensor-memory lane quarter
        const int ph = (warp - 4) >> 2;             // column half of G
        const int prow = 32 * pq + lane;
        const uint32_t tl = tm + ((uint32_t)(32 * pq) << 16);
        float *Lm = reinterpret_cast<float *>(smem_raw + kLm);
        float *Tm = reinterpret_cast<float *>(smem_raw + kTm);
        float *Zs = reinterpret_cast<float *>(smem_raw + kZs);
        // G(c) = [Q; K] K^T once chunk c is loaded (elected thread; the caller made sure G(c-1)
        // was read)
        auto issue_g = [&](int c) {
            const int s = c % kStages;
            if (!mbar_wait(&sm->full[s], (c / kStages) & 1, abort, p.err)) return;
            tc_fence_after();
            const uint32_t st = sb + s * kStage;
            mma_chain<8, true, true>(tm + kColG, dk(st), dk(st + 8192), id_g, false);
            mma_commit(&sm->g_done);
        };
        if (pe == 0) issue_g(0);
        for (int c = 0; c < nch; ++c) {
            const int s = c % kStages;
            const Gates *G = &sm->gt[s];
            // chunk c loaded and its gates ready; G(c) formed; the A buffer of this parity
            // free once A E(c - 2) is done
            if (pe == 0) {
                mbar_wait(&sm->full[s], (c / kStages) & 1, abort, p.err);
                mbar_wait(&sm->g_done, c & 1, abort, p.err);
                if (c >= 2) mbar_wait(&sm->ae_done[c & 1], ((c >> 1) - 1) & 1, abort, p.err);
            }
            if (named_sync_any(kBarPrep, kPrepT, *abort != 0)) break;
            tc_fence_after();
            {
                // rows 0-63 of G: Q K^T -> A tile (j <= t); rows 64-127: K K^T -> Lm (j < t);
                // columns j in [32 ph, 32 ph + 32).  The pair decay 2^(lam_t - lam_j) is the
                // row factor 2^(lam_t - lam_{j0}) of the 16-column block j0 times the column
                // factor cf_j, or (slow chunks) one exponential per element.
                const bool qrows = pq < 2;
                const int t = qrows ? prow : prow - 64;
                const float lt = G->lam[t], bt = qrows ? 1.f : G->bet[t];
                const bool empty = (pq & 1) == 0 && ph == 1;   // rows 0-31 x columns 32-63
                float v[32];
                if (!empty) tmem_ld32(tl + kColG + 32 * ph, v);
                if (G->slow) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int jj = 32 * ph + j;
                        const bool keep = !empty && (qrows ? jj <= t : jj < t);
                        v[j] = keep ? v[j] * bt * ex2(lt - G->lam[jj]) : 0.f;
                    }
                } else {
#pragma unroll
                    for (int bb = 0; bb < 2; ++bb) {
                        const int j0 = 32 * ph + 16 * bb;
                        const float rf = (j0 <= t) ? bt * ex2(lt - G->lam[j0]) : 0.f;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float4 c4 = *reinterpret_cast<const float4 *>(G->cf + j0 + 4 * q);
                            const float cc[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                const int jj = j0 + 4 * q + k, e = 16 * bb + 4 * q + k;
                                const bool keep = !empty && (qrows ? jj <= t : jj < t);
                                v[e] = keep ? v[e] * (rf * cc[k]) : 0.f;
                            }
                        }
                    }
                }
                if (qrows) {
                    const uint32_t abuf = sb + ((c & 1) ? kA1 : kA0);
                    st_row_bf16x16(abuf, t, 4 * ph, v);
                    st_row_bf16x16(abuf, t, 4 * ph + 2, v + 16);
                } else {
                    float4 *lr = reinterpret_cast<float4 *>(Lm + t * kTStride + 32 * ph);
#pragma unroll
                    for (int q = 0; q < 8; ++q) lr[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                }
            }
            fence_async_smem();
            tc_fence_before();
            named_sync(kBarPrep, kPrepT);
            // G is read: the next chunk's G may start
            if (pe == 0 && c + 1 < nch) issue_g(c + 1);
            // T = (I + Lm)^-1 (lower triangle)
            invert_unit_lower_rec<kBarPrep, kPrepT>(Lm, Tm, Zs, pe);
            // T diag(b), T diag(b g) as bf16 operands once W, U of chunk c - 1 are done
            if (c >= 1 && pe == 0) mbar_wait(&sm->wu_done, (c - 1) & 1, abort, p.err);
            if (named_sync_any(kBarPrep, kPrepT, *abort != 0)) break;
            {
                const int t = pe >> 2, j0 = 16 * (pe & 3);
                float v1[16], v2[16];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 tv = *reinterpret_cast<const float4 *>(Tm + t * kTStride + j0 + 4 * q);
                    const float4 b4 = *reinterpret_cast<const float4 *>(G->bet + j0 + 4 * q);
                    const float4 g4 = *reinterpret_cast<const float4 *>(G->bg + j0 + 4 * q);
                    const float tt[4] = {tv.x, tv.y, tv.z, tv.w}, bb[4] = {b4.x, b4.y, b4.z, b4.w},
                                gg[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float tj = (j0 + 4 * q + k <= t) ? tt[k] : 0.f;
                        v1[4 * q + k] = tj * bb[k];
                        v2[4 * q + k] = tj * gg[k];
                    }
                }
                st_row_bf16x16(sb + kTb, t, j0 >> 3, v1);
                st_row_bf16x16(sb + kTbg, t, j0 >> 3, v2);
            }
            fence_async_smem();
            named_sync(kBarPrep, kPrepT);
            if (pe == 0) {
                // W = T diag(b g) K into rows 64-127;  U = T diag(b) V (the V half) likewise,
                // once the chain has read W(c - 1) and U(c - 1)
                bool ok = true;
                if (c >= 1) {
                    ok = mbar_wait(&sm->w_free, (c - 1) & 1, abort, p.err) &&
                         mbar_wait(&sm->u_free, (c - 1) & 1, abort, p.err);
                }
                if (ok) {
                    tc_fence_after();
                    const uint32_t st = sb + s * kStage;
                    mma_chain<4, true, false>(tm + kColW, dk(sb + kTbg - 8192), dmn(st + 8192, 16384),
                                              id_w, false);
                    mma_chain<4, true, false>(tm + kColU, dk(sb + kTb - 8192), dmn(st + 32768, 8192),
                                              id_u, false);
                    mma_commit(&sm->wu_done);
                }
            }
        }
        // nothing this group issued may still write tensor memory when it is freed
        if (pe == 0) {
            mma_commit(&sm->g_done);   // completes phase nch (the G products took 0 .. nch-1)
            drain_wait(&sm->g_done, (uint32_t)nch & 1);
        }
        }
    } else if (warp >= 12) {
        // ------------------------------------------------------------ chain warps 12-15
        const int ce = threadIdx.x - 384;           // 0..127
        const int cq = warp & 3;                    // lane quarter
        const int row = 32 * cq + lane;             // d_k row of S^T; token of P / W / E
        const uint32_t tl = tm + ((uint32_t)(32 * cq) << 16);
        float Sr[kDV];   // S^T[row][32 vs + j]
        {
            const float *src = p.s_in ? p.s_in + slot + (size_t)(kDV * vs) * kD + row : nullptr;
#pragma unroll
            for (int j = 0; j < kDV; ++j) Sr[j] = src ? src[(size_t)j * kD] : 0.f;
            st_row32_mn(sb + kS, row, Sr);
            fence_async_smem();
        }
        // P(c) = [diag(g) Q; W] S^T  (rows 0-63: inter-chunk outputs, 64-127: W S^T), issued
        // by the elected thread once the S^T tile and the A operand are published
        auto issue_p = [&](int c) {
            tc_fence_after();
            mma_chain_ts<8>(tm + kColP + kDV * (c & 1), tm + kColQW + 64 * (c & 1), dmn(sb + kS, 8192),
                            id_p, false);
            mma_commit(&sm->p_done);
            if (TWO) mma_commit(&sm->p_done2[c & 1]);
            if (KDA) mbar_arrive(&sm->p_issued);
        };
        // two-pass: the prep warps wrote [diag(g) Q; W] of chunk c; the chain meets after the
        // elected thread saw it (which also orders the stage's gates before their reads)
        auto qw_wait = [&](int c) -> bool {
            return group_wait(&sm->qw_ready[c & 1], (c >> 1) & 1, ce == 0, kBarChain, kChainT, abort, p.err);
        };
        // [diag(g) Q; W] of chunk c into tensor memory as the A operand of P
        auto qw_step = [&](int c) -> bool {
            const int s = c % kStages;
            // the Q tile and the gates are read here: every thread observes the stage
            mbar_wait(&sm->full[s], (c / kStages) & 1, abort, p.err);
            if (!group_wait(&sm->wu_done, c & 1, ce == 0, kBarChain, kChainT, abort, p.err)) return false;
            tc_fence_after();
            const uint32_t dst = tl + kColQW + 64 * (c & 1);
            if (cq < 2) {
                const int t = row;
                const float gt = ex2(sm->gt[s].lam[t]);
                const uint32_t st = sb + s * kStage;
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    uint32_t w[32];
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        const uint4 x = scale_bf16x8(lds128(st + 16384 * h + sw128_off(t, ch)), gt);
                        w[4 * ch + 0] = x.x;
                        w[4 * ch + 1] = x.y;
                        w[4 * ch + 2] = x.z;
                        w[4 * ch + 3] = x.w;
                    }
                    tmem_st32(dst + 32 * h, w);
                }
            } else {
#pragma unroll 1
                for (int h = 0; h < 4; ++h) {
                    float f[32];
                    tmem_ld32(tl + kColW + 32 * h, f);
                    uint32_t w[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(f[2 * j], f[2 * j + 1]);
                    tmem_st16u(dst + 16 * h, w);
                }
            }
            tc_fence_before();
            named_sync(kBarChain, kChainT);
            if (ce == 0) mbar_arrive(&sm->w_free);
            return true;
        };
        bool ok = TWO ? qw_wait(0) : qw_step(0);
        if (ok && ce == 0) issue_p(0);
        // Iteration c: E of chunk c (lanes 64-127) and the outputs of chunk c - 1 (lanes 0-63);
        // the A operand of chunk c + 1 while dS(c) is formed; the state update and P(c + 1).
        // Iteration nch only writes the last outputs.
        for (int c = 0; c <= nch && ok; ++c) {
            const int s = c % kStages;
            const uint32_t par = c & 1;
            const bool cur = c < nch;
            // the stage's gates were observed in qw_step(c); read before the barrier below,
            // which precedes the stage's release (dS(c) is issued after it)
            // (KDA: the stage's per-row decay Gam_L of the chunk, d_k row `row`)
            float gL = 1.f;
            if (cur) {
                if constexpr (KDA) {
                    mbar_wait(&sm->full[s], (c / kStages) & 1, abort, p.err);
                    gL = reinterpret_cast<const float *>(smem_raw + s * kStage + GL::kGlOff)[row];
                } else {
                    gL = ex2(sm->gt[s].lam[kC - 1]);
                }
            }
            // P(c) done, and A E(c - 1) (which frees the E tiles and completes the outputs of
            // chunk c - 1; the tensor core ran it before P(c)): one meeting of the chain
            {
                if (ce == 0) {
                    if (cur) mbar_wait(&sm->p_done, par, abort, p.err);
                    if (c >= 1) mbar_wait(&sm->ae_done[(c - 1) & 1], ((c - 1) >> 1) & 1, abort, p.err);
                }
                if (named_sync_any(kBarChain, kChainT, *abort != 0)) break;
                tc_fence_after();
            }
            if (cq >= 2) {
                if (cur) {
                    // E = U - W S^T
                    const int t = row - 64;
                    const int L = sm->gt[s].len;
                    const float *lam = sm->gt[s].lam;
                    float y[32], uu[32];
                    tmem_ld32(tl + kColP + kDV * par, y);
                    tmem_ld32(tl + ((TWO && par) ? kColU2 : kColU) + kDV * (vs & 1), uu);
                    const float dec = (t < L) ? ex2(lam[kC - 1] - lam[t]) : 0.f;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float e = (t < L) ? uu[j] - y[j] : 0.f;
                        y[j] = e;
                        uu[j] = e * dec;
                    }
                    st_row32_mn(sb + kE, t, y);
                    st_row32_mn(sb + kEp, t, uu);
                    fence_async_smem();
                    tc_fence_before();
                    named_sync(kBarChainE, 64);
                    if (row == 64) {
                        mbar_arrive(TWO ? &sm->u_free2[par] : &sm->u_free);
                        tc_fence_after();
                        const uint32_t st = sb + s * kStage;
                        // dS^T = K^T E'   (E' = diag(dec) E)
                        // (KDA: K o 2^(lam_L - lam) in place of K, and E' = E)
                        mma_chain<4, false, false>(tm + kColDS, dmn(st + GL::kKlOff, GL::kKlHalf),
                                                   dmn(sb + kEp, 8192), id_ds, false);
                        mma_commit(&sm->ds_done);
                        mma_commit(&sm->empty[s]);
                        // rows 0-63 of P += A E  (the 64 rows after the A tile multiply into
                        // rows 64-127, already read)
                        // (two-pass: A(c) arrived before the chain saw qw_ready(c))
                        mma_chain<4, true, false>(tm + kColP + kDV * par, dk(sb + (par ? kA1 : kA0)),
                                                  dmn(sb + kE, 8192), id_ae, true);
                        mma_commit(&sm->ae_done[par]);
                    }
                }
            } else if (c >= 1) {
                // outputs of chunk c - 1: rows 0-63 of P (lanes 0-63), the slice's 32 columns

                const int t = row;
                const int t0 = tb + kC * (c - 1);
                const int L = min(kC, te - t0);
                float v[32];
                tmem_ld32(tl + kColP + kDV * ((c - 1) & 1), v);
                if (t < L) {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.o + ((size_t)bh * p.T + t0 + t) * kD + kDV * vs);
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
            }
            if (!TWO && c + 1 < nch && !qw_step(c + 1)) break;
            if (!cur) continue;
            // ---- state: S^T <- g_{L-1} S^T + dS^T; bf16 copy for the next chunk (two-pass: one
            // meeting also covers the next chunk's A operand of P)
            if constexpr (TWO) {
                if (ce == 0) {
                    if (c + 1 < nch) mbar_wait(&sm->qw_ready[(c + 1) & 1], ((c + 1) >> 1) & 1, abort, p.err);
                    mbar_wait(&sm->ds_done, par, abort, p.err);
                }
                if (named_sync_any(kBarChain, kChainT, *abort != 0)) break;
            } else {
                if (!group_wait(&sm->ds_done, par, ce == 0, kBarChain, kChainT, abort, p.err)) break;
            }
            tc_fence_after();
            const bool last = (c + 1 == nch);
            {
                float d[32];
                tmem_ld32(tl + kColDS, d);
#pragma unroll
                for (int j = 0; j < kDV; ++j) Sr[j] = fmaf(gL, Sr[j], d[j]);
            }
            if (last) {
                if (p.s_out) {
                    float *dst = p.s_out + slot + (size_t)(kDV * vs) * kD + row;
#pragma unroll
                    for (int j = 0; j < kDV; ++j) dst[(size_t)j * kD] = Sr[j];
                }
            } else {
                st_row32_mn(sb + kS, row, Sr);
                fence_async_smem();
            }
            tc_fence_before();
            named_sync(kBarChain, kChainT);
            if (ce == 0 && !last) issue_p(c + 1);
        }
        // nothing this group issued may still write tensor memory when it is freed
        if (ce == 0) {
            mma_commit(&sm->p_done);
            drain_wait(&sm->p_done, (uint32_t)nch & 1);
        }
        if (row == 64) {
            mma_commit(&sm->ds_done);
            drain_wait(&sm->ds_done, (uint32_t)nch & 1);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tm, kTmemCols);
    }
}

}  // namespace

bool prefill_gdn_selected(int mode, int BH, bool packed) {
    // Dense calls whose d_v slices fill 64 to 148 SMs (one wave): there the single pass is as
    // fast as the segmented kernels and moves the algorithmic bytes once (no workspace, no
    // second pass over k and v).  Fewer heads take the segmented kernels (which split long
    // sequences over more SMs), more heads one CTA per head; packed sequences take the
    // per-sequence kernel.
    return mode == LA_MODE_GATED_DELTA && !packed && BH * kNS >= 64 && BH * kNS <= 148;
}

size_t prefill_gdn_workspace_bytes(int BH, int T) {
    return sizeof(__nv_bfloat16) * (size_t)kImgHalves * (size_t)BH * (size_t)((T + kC - 1) / kC);
}

bool prefill_kda2_selected(int mode, int BH, bool packed) {
    // The same head-row range as the gated delta rule; KDA runs here only in the two-pass
    // variant (with a workspace of prefill_kda2_workspace_bytes), else on the segmented kernels.
    return mode == LA_MODE_KDA && !packed && BH * kNS >= 64 && BH * kNS <= 148;
}

size_t prefill_kda2_workspace_bytes(int BH, int T) {
    return (size_t)kKdaRec * (size_t)BH * (size_t)((T + kC - 1) / kC);
}

// With a workspace of at least prefill_gdn_workspace_bytes (dense calls), pass 1 forms every
// chunk's A, T diag(b), T diag(b g) at once and the chain kernel reads them (two-pass);
// otherwise the single pass forms them itself.
namespace {
cudaError_t launch_gdn(const PrefillArgs &a, void *workspace, size_t workspace_bytes, const ConvSpec *cs) {
    const int BH = a.cu ? a.H : a.B * a.H;
    const bool kda = a.mode == LA_MODE_KDA;   // (two-pass only; its gates go to pass 1)
    GdnParams p;
    memset(&p, 0, sizeof(p));
    const uint64_t row_pitch = kD * 2, head_pitch = (uint64_t)a.T * kD * 2;
    if (!make_tmap_3d(&p.tq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kD, a.T, BH, row_pitch,
                      head_pitch, 64, kC, true) ||
        !make_tmap_3d(&p.tk, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kD, a.T, BH, row_pitch,
                      head_pitch, 64, kC, true) ||
        !make_tmap_3d(&p.tv, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kD, a.T, BH, row_pitch,
                      head_pitch, 64, kC, true))
        return cudaErrorInvalidValue;
    p.gate = kda ? nullptr : a.gate;
    p.beta = a.beta;
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.s_in = a.init_state ? a.state : nullptr;
    p.s_out = a.state;
    p.seq_stride = a.cu ? (long long)a.H * kD * kD : 0;
    p.cu = a.cu;
    p.T = a.T;
    p.BH = BH;
    p.err = device_error_word();
    const int units = a.cu ? a.nseq * a.H : BH;
    const bool two = !a.cu && workspace && (reinterpret_cast<uintptr_t>(workspace) & 15u) == 0 &&
                     workspace_bytes >= (kda ? prefill_kda2_workspace_bytes(BH, a.T)
                                             : prefill_gdn_workspace_bytes(BH, a.T));
    if (cs && !two) return cudaErrorInvalidValue;   // the fused convolution lives in pass 1
    if (kda && (!two || cs || (reinterpret_cast<uintptr_t>(a.gate) & 15u) != 0)) return cudaErrorInvalidValue;
    cudaError_t e;
    if (two) {
        const int nch = (a.T + kC - 1) / kC;
        p.img = static_cast<const __nv_bfloat16 *>(workspace);
        p.nchunks = nch;
        FacConv fc;
        memset(&fc, 0, sizeof(fc));
        if (cs) {
            for (int z = 0; z < 3; ++z) {
                fc.x[z] = static_cast<const __nv_bfloat16 *>(cs->x[z]);
                fc.w[z] = cs->w[z];
            }
            fc.win_in = static_cast<const __nv_bfloat16 *>(cs->win_in);
            fc.win_out = static_cast<__nv_bfloat16 *>(cs->win_out);
            fc.y = static_cast<__nv_bfloat16 *>(cs->y);
            fc.B = a.B;
            fc.H = a.H;
            fc.width = cs->width;
            fc.fqk = cs->fqk;
            fc.fv = cs->fv;
        }
        auto fac = cs ? gdn_chunk_factors_kernel<true> : gdn_chunk_factors_kernel<false>;
        const uint32_t fbytes = kda ? kkBytes : cs ? FacLay<true>::kBytes : FacLay<false>::kBytes;
        e = kda ? cudaFuncSetAttribute(kda_chunk_factors_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)fbytes)
                : cudaFuncSetAttribute(fac, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fbytes);
        if (e != cudaSuccess) return e;
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return cudaErrorUnknown;
        const int total = BH * nch;
        const int grid = total < 2 * sms ? total : 2 * sms;
        timer_begin(a.stream);
        if (kda)
            kda_chunk_factors_kernel<<<(unsigned)grid, kFacT, fbytes, a.stream>>>(
                static_cast<const __nv_bfloat16 *>(a.q), static_cast<const __nv_bfloat16 *>(a.k), a.gate, a.beta,
                a.T, nch, total, static_cast<uint8_t *>(workspace));
        else
            fac<<<(unsigned)grid, kFacT, fbytes, a.stream>>>(
                static_cast<const __nv_bfloat16 *>(a.q), static_cast<const __nv_bfloat16 *>(a.k), a.gate, a.beta,
                a.T, nch, total, static_cast<__nv_bfloat16 *>(workspace), fc);
        timer_end(a.stream);
        note_launches(1);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    auto kern = kda ? gdn_prefill_kernel<kTwoKda> : two ? gdn_prefill_kernel<kTwoGdn> : gdn_prefill_kernel<kSingle>;
    const uint32_t bytes = kda ? GLay<kTwoKda>::kBytes : two ? GLay<kTwoGdn>::kBytes : GLay<kSingle>::kBytes;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    timer_begin(a.stream);
    kern<<<units * kNS, kThreads, bytes, a.stream>>>(p);
    timer_end(a.stream);
    note_launches(1);
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_prefill_gdn(const PrefillArgs &a, void *workspace, size_t workspace_bytes) {
    return launch_gdn(a, workspace, workspace_bytes, nullptr);
}

// KDA (mode 3) in the two-pass variant: the caller checked prefill_kda2_selected, the
// workspace size and a 16-byte aligned gate tensor.
cudaError_t launch_prefill_kda2(const PrefillArgs &a, void *workspace, size_t workspace_bytes) {
    return launch_gdn(a, workspace, workspace_bytes, nullptr);
}

// Pass 1 convolves the projections as it loads them and writes the convolved q, k, v
// (a.q, a.k, a.v point into cs.y); pass 2 reads those.
cudaError_t launch_prefill_gdn_conv(const PrefillArgs &a, const ConvSpec &cs, void *workspace,
                                    size_t workspace_bytes) {
    return launch_gdn(a, workspace, workspace_bytes, &cs);
}

}  // namespace la

// conv.cu -- the short causal depthwise convolution in front of q, k and v
// (la_short_conv, la_short_conv_step).
//
// Lesson page "Linear attention and hybrids", section "Hybrids of 2025: Qwen3-Next and
// Kimi Linear": Gated DeltaNet and KDA layers mix each token with the three before it
// by a causal depthwise convolution over time, kernel width 4.  Per channel c, with the
// carried window x_{-1}, x_{-2}, ... in front of the sequence:
//
//   u_t[c] = sum_{i < W} w[c][i] x_{t-(W-1)+i}[c],   optionally  u <- u * sigmoid(u),
//   optionally every head's row  u <- u / sqrt(sum_d u^2 + 1e-6),
//
// read token-major [B, T, H*d] and written head-major [B, H, T, d], the layout of the
// attention kernels.  The work is a stream (one read and one write of every element, W
// multiply-adds and an activation each), so the kernel is built for HBM bandwidth:
//   - a thread owns 8 channels (one 16-byte bf16 vector) of one batch row and walks a
//     run of kRun consecutive tokens, keeping the last W-1 inputs in registers;
//   - its input rows arrive through a private ring of kDepth slots in shared memory
//     filled by cp.async, kDepth rows ahead of use, so that the bytes in flight cost no
//     registers (a register-staged version with the same arithmetic reached 60% of the
//     bandwidth of this one);
//   - tokens are taken in pairs, so the two rows' shuffle reductions of the head norm
//     and their activations interleave instead of running as one long dependent chain;
//   - consecutive threads own consecutive channel groups: each warp reads 512
//     contiguous bytes per token, and a head's d/8 threads are adjacent lanes.
// The W-1 tokens before a run are re-read with plain loads (from L2 in practice: the
// neighbouring run is the neighbouring block).
// SiLU: for bf16 output the sigmoid is 1/2 + tanh(u/2)/2 with the tanh.approx
// instruction, whose absolute error (below 2^-11) moves the output by at most
// |u| 2^-12, under half a bf16 step of the row's large entries; it keeps the kernel at
// the bandwidth bound.  fp32 output uses u / (1 + expf(-u)).
#include "la_internal.cuh"

namespace la {
namespace {

constexpr int kConvThreads = 256;
constexpr int kRun = 64;     // tokens per thread
constexpr int kDepth = 8;    // ring slots (rows in flight) per thread; even
constexpr float kL2Eps = 1e-6f;

struct Vec8 {
    float v[8];
};

// 8 channels as they sit in memory: one 16-byte vector of bf16, or two of fp32.  Tiles
// stay in this form in registers (half the registers for bf16) and are widened to fp32
// where they are used.
template <typename IO>
struct Raw;
template <>
struct Raw<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float *p) {
        a = *reinterpret_cast<const float4 *>(p);
        b = *reinterpret_cast<const float4 *>(p + 4);
    }
    __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ void store(float *p) const {
        *reinterpret_cast<float4 *>(p) = a;
        *reinterpret_cast<float4 *>(p + 4) = b;
    }
    __device__ __forceinline__ Vec8 f32() const { return Vec8{{a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w}}; }
};
template <>
struct Raw<__nv_bfloat16> {
    uint4 r;
    __device__ __forceinline__ void load(const __nv_bfloat16 *p) { r = *reinterpret_cast<const uint4 *>(p); }
    __device__ __forceinline__ void zero() { r = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ void store(__nv_bfloat16 *p) const { *reinterpret_cast<uint4 *>(p) = r; }
    __device__ __forceinline__ Vec8 f32() const {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
        Vec8 o;
#pragma unroll
        for (int j = 0; j < 4; ++j) {   // bf16 -> fp32 is exact: the high half of the word
            o.v[2 * j] = __uint_as_float(w[j] << 16);
            o.v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
        }
        return o;
    }
};

__device__ __forceinline__ void store8(float *p, const Vec8 &x) {
    *reinterpret_cast<float4 *>(p) = make_float4(x.v[0], x.v[1], x.v[2], x.v[3]);
    *reinterpret_cast<float4 *>(p + 4) = make_float4(x.v[4], x.v[5], x.v[6], x.v[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16 *p, const Vec8 &x) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(x.v[2 * j], x.v[2 * j + 1]);
        w[j] = *reinterpret_cast<const uint32_t *>(&h);
    }
    *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ Vec8 zero8() { return Vec8{{0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}}; }

__device__ __forceinline__ float silu_fast(float u) {   // u sigmoid(u), sigmoid via tanh.approx
    float t;
    const float h = 0.5f * u;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
    return fmaf(h, t, h);
}

// Activation and per-head row norm of two tokens' 8 channels, interleaved.  NL lanes
// (d / 8, adjacent and aligned) hold one head's row; `mask` names them.
template <typename IO, bool SILU, bool L2, int NL>
__device__ __forceinline__ void activate2(Vec8 &u0, Vec8 &u1, unsigned mask) {
    if (SILU) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if constexpr (sizeof(IO) == 2) {
                u0.v[j] = silu_fast(u0.v[j]);
                u1.v[j] = silu_fast(u1.v[j]);
            } else {
                u0.v[j] = u0.v[j] / (1.f + expf(-u0.v[j]));
                u1.v[j] = u1.v[j] / (1.f + expf(-u1.v[j]));
            }
        }
    }
    if (L2) {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            s0 = fmaf(u0.v[j], u0.v[j], s0);
            s1 = fmaf(u1.v[j], u1.v[j], s1);
        }
#pragma unroll
        for (int off = NL / 2; off > 0; off >>= 1) {
            s0 += __shfl_xor_sync(mask, s0, off);
            s1 += __shfl_xor_sync(mask, s1, off);
        }
        const float r0 = rsqrtf(s0 + kL2Eps), r1 = rsqrtf(s1 + kL2Eps);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            u0.v[j] *= r0;
            u1.v[j] *= r1;
        }
    }
}

template <int NL>
__device__ __forceinline__ unsigned head_mask(int lane) {
    return (NL == 32 ? 0xffffffffu : ((1u << NL) - 1u)) << (lane & ~(NL - 1));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int W>
__device__ __forceinline__ void load_taps(const float *w, int c0, float (&wr)[W][8]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        if constexpr (W == 4) {   // one 16-byte row of taps per channel
            const float4 a = *reinterpret_cast<const float4 *>(w + (size_t)(c0 + j) * 4);
            wr[0][j] = a.x; wr[1][j] = a.y; wr[2][j] = a.z; wr[3][j] = a.w;
        } else {
#pragma unroll
            for (int i = 0; i < W; ++i) wr[i][j] = w[(size_t)(c0 + j) * W + i];
        }
    }
}

// u = sum_i wr[i] * window[i] (i < W-1) + wr[W-1] * x; then the window shifts by one.
template <int W, typename IO>
__device__ __forceinline__ Vec8 conv_step(const float (&wr)[W][8], Raw<IO> (&win)[W > 1 ? W - 1 : 1],
                                          const Raw<IO> &xr) {
    const Vec8 x = xr.f32();
    Vec8 u;
#pragma unroll
    for (int j = 0; j < 8; ++j) u.v[j] = wr[W - 1][j] * x.v[j];
#pragma unroll
    for (int i = 0; i < W - 1; ++i) {
        const Vec8 p = win[i].f32();
#pragma unroll
        for (int j = 0; j < 8; ++j) u.v[j] = fmaf(wr[i][j], p.v[j], u.v[j]);
    }
    if (W > 1) {
#pragma unroll
        for (int i = 0; i + 1 < W - 1; ++i) win[i] = win[i + 1];
        win[W > 1 ? W - 2 : 0] = xr;
    }
    return u;
}

// Offset i of a packed sequence table, clamped to [0, T] (a bad table stays in bounds;
// the window pass reports it).
__device__ __forceinline__ int cu_at(const int *cu, int i, int T) { return min(max(cu[i], 0), T); }

// Three CTAs per SM for bf16 (80 registers); fp32 rows take twice the registers.
// PACKED: x is [T][C] holding N sequences back to back (sequence s = tokens cu[s] ..
// cu[s+1]); a thread's run may cross sequence starts, where its window restarts from
// that sequence's carried window.  The windows after the call are written by
// packed_window_kernel.
template <int W, typename IO, bool SILU, bool L2, int NL, bool PACKED>
__global__ void __launch_bounds__(kConvThreads, sizeof(IO) == 2 ? 3 : 2)
short_conv_kernel(int T, int H, int nrun, long long total, const IO *__restrict__ x,
                  const float *__restrict__ w, const IO *__restrict__ win_in,
                  IO *__restrict__ win_out, IO *__restrict__ y, const int *__restrict__ cu,
                  int N) {
    constexpr int d = NL * 8;
    constexpr int kVec = sizeof(Raw<IO>) / 16;    // 16-byte pieces per 8 channels
    extern __shared__ uint4 ring[];               // [kDepth][kConvThreads][kVec]
    const long long idx = (long long)blockIdx.x * kConvThreads + threadIdx.x;
    if (idx >= total) return;   // whole heads only: total is a multiple of d / 8
    const int C = H * d, G = C >> 3;
    const int g = (int)(idx % G);
    const long long rest = idx / G;
    const int run = (int)(rest % nrun);
    const long long b = rest / nrun;
    const int c0 = 8 * g, h = c0 / d, dd = c0 % d;
    const unsigned mask = head_mask<NL>(threadIdx.x & 31);

    const IO *xb = x + (size_t)b * T * C + c0;
    const int t0 = run * kRun;
    const int t1 = min(T, t0 + kRun);
    // ring slot k of this thread; rows t0 + k, t0 + k + kDepth, ... pass through it
    const uint32_t slot0 = (uint32_t)__cvta_generic_to_shared(ring) + threadIdx.x * 16 * kVec;
    constexpr uint32_t kSlotStride = kConvThreads * 16 * kVec;
    auto fetch = [&](int k, int t) {
#pragma unroll
        for (int p = 0; p < kVec; ++p)
            cp_async16(slot0 + k * kSlotStride + 16 * p, reinterpret_cast<const uint4 *>(xb + (size_t)t * C) + p);
    };
    // one commit group per pair of rows
#pragma unroll
    for (int k = 0; k < kDepth; k += 2) {
        if (t0 + k < t1) fetch(k, t0 + k);
        if (t0 + k + 1 < t1) fetch(k + 1, t0 + k + 1);
        cp_async_commit();
    }
    float wr[W][8];
    load_taps<W>(w, c0, wr);
    constexpr int WM = W > 1 ? W - 1 : 1;
    Raw<IO> win[WM];
    // packed: the sequence sq holding the current token, its first token a, and the next
    // sequence start nb
    int sq = 0, a = 0, nb = T;
    // the window in front of token t: rows of the current sequence, else its carried
    // window (index W-1 + row - a, within [0, W-2] because t >= a), else zeros
    auto load_window = [&](int t, const IO *wsrc) {
#pragma unroll
        for (int i = 0; i < W - 1; ++i) {
            const int row = t - (W - 1) + i;
            if (row >= a) win[i].load(xb + (size_t)row * C);
            else if (wsrc) win[i].load(wsrc + (size_t)((W - 1) + row - a) * C);
            else win[i].zero();
        }
    };
    if constexpr (PACKED) {
        int lo = 0, hi = N - 1;   // the last sequence starting at or before t0
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (cu_at(cu, mid, T) <= t0) lo = mid;
            else hi = mid - 1;
        }
        sq = lo;
        a = min(cu_at(cu, sq, T), t0);
        nb = max(cu_at(cu, sq + 1, T), t0 + 1);
        load_window(t0, win_in ? win_in + (size_t)sq * (W - 1) * C + c0 : nullptr);
    } else {
#pragma unroll
        for (int i = 0; i < W - 1; ++i) {
            const int t = t0 - (W - 1) + i;
            if (t >= 0) win[i].load(xb + (size_t)t * C);
            else if (win_in) win[i].load(win_in + ((size_t)b * (W - 1) + (W - 1) + t) * C + c0);
            else win[i].zero();
        }
    }
    // packed: token t starts a later sequence; move to it and restart the window
    auto enter = [&](int t) {
        while (sq + 1 < N && cu_at(cu, sq + 1, T) <= t) ++sq;
        a = min(cu_at(cu, sq, T), t);
        nb = (sq + 1 < N) ? max(cu_at(cu, sq + 1, T), t + 1) : T;
        load_window(t, win_in ? win_in + (size_t)sq * (W - 1) * C + c0 : nullptr);
    };
    IO *yb = y + (((size_t)b * H + h) * T) * d + dd;
    for (int tb = t0; tb < t1; tb += kDepth) {
#pragma unroll
        for (int k = 0; k < kDepth; k += 2) {
            const int t = tb + k;
            if (t < t1) {   // uniform across the head's lanes (same run)
                cp_async_wait<kDepth / 2 - 1>();   // the pair (t, t+1) has landed
                const bool has1 = t + 1 < t1;
                Raw<IO> x0, x1;
                const uint4 *r0 = ring + (size_t)(k * kConvThreads + threadIdx.x) * kVec;
                const uint4 *r1 = r0 + kConvThreads * kVec;
                x0 = *reinterpret_cast<const Raw<IO> *>(r0);
                x1 = *reinterpret_cast<const Raw<IO> *>(r1);
                // The second row of a pair past the run's end is stale slot contents:
                // computed but never stored (a conditional step would cost registers), so
                // the window registers are not the carried window at the end.
                if (PACKED && t >= nb) enter(t);
                Vec8 u0 = conv_step<W, IO>(wr, win, x0);
                if (PACKED && has1 && t + 1 >= nb) enter(t + 1);
                Vec8 u1 = conv_step<W, IO>(wr, win, x1);
                // refill both slots with the rows kDepth further on
                if (t + kDepth < t1) fetch(k, t + kDepth);
                if (t + 1 + kDepth < t1) fetch(k + 1, t + 1 + kDepth);
                cp_async_commit();
                activate2<IO, SILU, L2, NL>(u0, u1, mask);
                store8(yb + (size_t)t * d, u0);
                if (has1) store8(yb + (size_t)(t + 1) * d, u1);
            }
        }
    }
    // The carried window after the sequence, the last W-1 rows of [win_in; x]: written
    // by the run-0 thread, the only one that reads win_in, so that win_out may be win_in
    // itself.
    if (!PACKED && win_out && run == 0) {
#pragma unroll
        for (int i = 0; i < W - 1; ++i) {
            const int t = T - (W - 1) + i;
            Raw<IO> r;
            if (t >= 0) r.load(xb + (size_t)t * C);
            else if (win_in) r.load(win_in + ((size_t)b * (W - 1) + (W - 1) + t) * C + c0);
            else r.zero();
            r.store(win_out + ((size_t)b * (W - 1) + i) * C + c0);
        }
    }
    cp_async_wait<0>();   // no copy may still target shared memory at exit
}

// Packed sequences: window_out[s] = the last W-1 rows of [window_in[s]; x[cu[s] ..
// cu[s+1]]], one thread per (sequence, 8 channels).  Runs after the main pass (stream
// order), so window_out may be window_in: each thread reads its rows before writing.
// A decreasing or out-of-range offset is reported in the failure word.
template <int W, typename IO>
__global__ void __launch_bounds__(kConvThreads)
packed_window_kernel(int T, int C, int N, const int *__restrict__ cu, const IO *__restrict__ x,
                     const IO *__restrict__ win_in, IO *__restrict__ win_out, unsigned *err) {
    const long long idx = (long long)blockIdx.x * kConvThreads + threadIdx.x;
    const int G = C >> 3;
    if (idx >= (long long)N * G) return;
    const int sq = (int)(idx / G), c0 = 8 * (int)(idx % G);
    const int ra = cu[sq], rb = cu[sq + 1];
    const int a = cu_at(cu, sq, T), b = max(cu_at(cu, sq + 1, T), a);
    if ((ra != a || rb != b) && err) atomicOr(err, (unsigned)kErrBadInput);
    if (W == 1 || !win_out) return;
    constexpr int WM = W > 1 ? W - 1 : 1;
    Raw<IO> r[WM];
    const IO *wsrc = win_in ? win_in + (size_t)sq * (W - 1) * C + c0 : nullptr;
#pragma unroll
    for (int i = 0; i < W - 1; ++i) {
        const int row = b - (W - 1) + i;
        if (row >= a) r[i].load(x + (size_t)row * C + c0);
        else if (wsrc) r[i].load(wsrc + (size_t)((W - 1) + row - a) * C);
        else r[i].zero();
    }
#pragma unroll
    for (int i = 0; i < W - 1; ++i) r[i].store(win_out + ((size_t)sq * (W - 1) + i) * C + c0);
}

template <int W, typename IO, bool SILU, bool L2, int NL>
__global__ void __launch_bounds__(kConvThreads)
short_conv_step_kernel(int H, long long total, const IO *__restrict__ x,
                       const float *__restrict__ w, IO *__restrict__ window, IO *__restrict__ y) {
    constexpr int d = NL * 8;
    const long long idx = (long long)blockIdx.x * kConvThreads + threadIdx.x;
    if (idx >= total) return;
    const int C = H * d, G = C >> 3;
    const int g = (int)(idx % G);
    const long long n = idx / G;
    const int c0 = 8 * g;
    const unsigned mask = head_mask<NL>(threadIdx.x & 31);
    float wr[W][8];
    load_taps<W>(w, c0, wr);
    constexpr int WM = W > 1 ? W - 1 : 1;
    Raw<IO> win[WM];
    IO *wn = W > 1 ? window + (size_t)n * (W - 1) * C + c0 : nullptr;
#pragma unroll
    for (int i = 0; i < W - 1; ++i) win[i].load(wn + (size_t)i * C);
    Raw<IO> xr;
    xr.load(x + (size_t)n * C + c0);
    Vec8 u = conv_step<W, IO>(wr, win, xr);
#pragma unroll
    for (int i = 0; i < W - 1; ++i) win[i].store(wn + (size_t)i * C);
    Vec8 none = zero8();
    activate2<IO, SILU, L2, NL>(u, none, mask);
    store8(y + (size_t)n * C + c0, u);   // [N, H, d] and [N, H*d] coincide
}

template <int W, typename IO, bool SILU, bool L2, int NL>
cudaError_t launch_conv(const ConvArgs &a) {
    const int C = a.H * a.d, G = C / 8;
    if (a.step) {
        const long long total = (long long)a.B * G;
        const unsigned blocks = (unsigned)((total + kConvThreads - 1) / kConvThreads);
        timer_begin(a.stream);
        short_conv_step_kernel<W, IO, SILU, L2, NL><<<blocks, kConvThreads, 0, a.stream>>>(
            a.H, total, static_cast<const IO *>(a.x), a.w, static_cast<IO *>(a.win_out),
            static_cast<IO *>(a.y));
        timer_end(a.stream);
    } else if (a.cu) {
        const int nrun = (a.T + kRun - 1) / kRun;
        const long long total = (long long)nrun * G;
        const unsigned blocks = (unsigned)((total + kConvThreads - 1) / kConvThreads);
        const int smem = kDepth * kConvThreads * (int)sizeof(Raw<IO>);
        auto kern = short_conv_kernel<W, IO, SILU, L2, NL, true>;
        cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (err != cudaSuccess) return err;
        if (a.T > 0) {
            timer_begin(a.stream);
            kern<<<blocks, kConvThreads, smem, a.stream>>>(
                a.T, a.H, nrun, total, static_cast<const IO *>(a.x), a.w,
                static_cast<const IO *>(a.win_in), nullptr, static_cast<IO *>(a.y), a.cu, a.B);
            timer_end(a.stream);
            note_launches(1);
            err = cudaGetLastError();
            if (err != cudaSuccess) return err;
        }
        {   // the window pass (also the check of the offsets table)
            const long long nt = (long long)a.B * G;
            timer_begin(a.stream);
            packed_window_kernel<W, IO><<<(unsigned)((nt + kConvThreads - 1) / kConvThreads),
                                          kConvThreads, 0, a.stream>>>(
                a.T, C, a.B, a.cu, static_cast<const IO *>(a.x), static_cast<const IO *>(a.win_in),
                static_cast<IO *>(a.win_out), device_error_word());
            timer_end(a.stream);
            note_launches(1);
        }
        return cudaGetLastError();
    } else {
        const int nrun = (a.T + kRun - 1) / kRun;
        const long long total = (long long)a.B * nrun * G;
        const unsigned blocks = (unsigned)((total + kConvThreads - 1) / kConvThreads);
        const int smem = kDepth * kConvThreads * (int)sizeof(Raw<IO>);
        auto kern = short_conv_kernel<W, IO, SILU, L2, NL, false>;
        cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (err != cudaSuccess) return err;
        timer_begin(a.stream);
        kern<<<blocks, kConvThreads, smem, a.stream>>>(
            a.T, a.H, nrun, total, static_cast<const IO *>(a.x), a.w,
            static_cast<const IO *>(a.win_in), static_cast<IO *>(a.win_out),
            static_cast<IO *>(a.y), nullptr, 0);
        timer_end(a.stream);
    }
    note_launches(1);
    return cudaGetLastError();
}

template <int W, typename IO, bool SILU, bool L2>
cudaError_t launch_head(const ConvArgs &a) {
    return a.d == 128 ? launch_conv<W, IO, SILU, L2, 16>(a) : launch_conv<W, IO, SILU, L2, 8>(a);
}

template <int W, typename IO>
cudaError_t launch_flags(const ConvArgs &a) {
    if (a.silu) return a.l2norm ? launch_head<W, IO, true, true>(a) : launch_head<W, IO, true, false>(a);
    return a.l2norm ? launch_head<W, IO, false, true>(a) : launch_head<W, IO, false, false>(a);
}

template <typename IO>
cudaError_t launch_width(const ConvArgs &a) {
    switch (a.width) {
        case 1: return launch_flags<1, IO>(a);
        case 2: return launch_flags<2, IO>(a);
        case 3: return launch_flags<3, IO>(a);
        case 4: return launch_flags<4, IO>(a);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_short_conv(const ConvArgs &a) {
    return a.dtype == LA_BF16 ? launch_width<__nv_bfloat16>(a) : launch_width<float>(a);
}

}  // namespace la

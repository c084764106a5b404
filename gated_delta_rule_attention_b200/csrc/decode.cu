// decode.cu -- one recurrent token for N sequences x H heads (la_decode_step).
//
// The recurrent form of "Linear attention and hybrids" (section "Three forms of one
// computation"), with the decay of section "Memory must forget" and the Gated DeltaNet
// update of section "The delta rule and Gated DeltaNet".  Per head the state row
// s_j (row j of S, d_k floats) evolves independently of every other row:
//
//   mode 2:  e_j = b (v_j - a s_j.k);   s_j <- a s_j + e_j k;   o_j = a (s_j.q) + e_j (k.q)
//   mode 3:  the same with the row first decayed per channel, s_j <- s_j o a (Kimi Delta
//            Attention: Diag(a) for the scalar a), then a = 1
//   mode 1:  s_j <- a s_j + v_j k;                              o_j = a (s_j.q) + v_j (k.q)
//   mode 0:  s_j <- s_j + v_j phi(k);  z <- z + phi(k);
//            o_j = (s_j.phi(q) + v_j phi(k).phi(q)) / (z_new . phi(q))
//
// (s_j on the right-hand sides is the old row; the o_j expressions are S_t q_t
// expanded so that both dot products read the row once.)  The step streams the fp32
// state once in and once out: 2 d_k d_v 4 bytes per head, a pure HBM-bandwidth
// problem.  One CTA per (sequence, head), 8 warps; each warp owns d_v / 8 contiguous
// rows, holds d_k / 32 floats of a row per lane, and keeps ROWS rows in flight so that
// every SM has enough bytes outstanding to cover DRAM latency.
#include "la_internal.cuh"

namespace la {
namespace {

constexpr int kDecodeThreads = 256;
constexpr int kDecodeWarps = kDecodeThreads / 32;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

template <int VEC>
struct Row;
template <>
struct Row<4> {
    float x[4];
    __device__ __forceinline__ void load(const float *p) {
        const float4 t = *reinterpret_cast<const float4 *>(p);
        x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    }
    __device__ __forceinline__ void store(float *p) const {
        *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
    }
};
template <>
struct Row<2> {
    float x[2];
    __device__ __forceinline__ void load(const float *p) {
        const float2 t = *reinterpret_cast<const float2 *>(p);
        x[0] = t.x; x[1] = t.y;
    }
    __device__ __forceinline__ void store(float *p) const {
        *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]);
    }
};

template <int MODE, int DK, int DV, typename IO>
__global__ void __launch_bounds__(kDecodeThreads)
decode_kernel(const IO *__restrict__ q, const IO *__restrict__ k, const IO *__restrict__ v,
              const float *__restrict__ gate, const float *__restrict__ beta,
              float *__restrict__ state, float *__restrict__ z, IO *__restrict__ o,
              int gate_heads) {
    constexpr int VEC = DK / 32;
    constexpr int RPW = DV / kDecodeWarps;       // rows per warp: 16 or 8
    constexpr int ROWS = RPW < 4 ? RPW : 4;      // rows in flight per warp
    static_assert(RPW % ROWS == 0, "rows per warp must be a multiple of ROWS");

    __shared__ float o_s[DV];
    const size_t nh = blockIdx.x;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;

    float qv[VEC], kv[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
        qv[e] = to_f32(q[nh * DK + lane * VEC + e]);
        kv[e] = to_f32(k[nh * DK + lane * VEC + e]);
        if (MODE == 0) {
            qv[e] = feature_phi(qv[e]);
            kv[e] = feature_phi(kv[e]);
        }
    }
    constexpr bool kDelta = (MODE == 2 || MODE == 3);
    const float a = (MODE == 0 || MODE == 3 || gate == nullptr) ? 1.f
                                                                 : gate[gate_heads ? nh % gate_heads : nh];
    const float b = kDelta ? beta[nh] : 0.f;
    float av[VEC];   // mode 3: this lane's channel decays
#pragma unroll
    for (int e = 0; e < VEC; ++e) av[e] = (MODE == 3 && gate) ? gate[nh * DK + lane * VEC + e] : 1.f;
    float kq = 0.f;
#pragma unroll
    for (int e = 0; e < VEC; ++e) kq = fmaf(kv[e], qv[e], kq);
    kq = warp_sum(kq);

    float inv_den = 1.f;
    if (MODE == 0) {
        float zn[VEC], zq = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            zn[e] = z[nh * DK + lane * VEC + e] + kv[e];
            zq = fmaf(zn[e], qv[e], zq);
        }
        inv_den = 1.f / warp_sum(zq);
        __syncthreads();  // every warp has read the old z before warp 0 overwrites it
        if (warp == 0) {
#pragma unroll
            for (int e = 0; e < VEC; ++e) z[nh * DK + lane * VEC + e] = zn[e];
        }
    }

    float *S = state + nh * (size_t)DV * DK;
    const IO *vh = v + nh * DV;
    const int row0 = warp * RPW;
#pragma unroll 1
    for (int rr = 0; rr < RPW; rr += ROWS) {
        Row<VEC> s[ROWS];
        float vj[ROWS];
#pragma unroll
        for (int j = 0; j < ROWS; ++j) {
            s[j].load(S + (size_t)(row0 + rr + j) * DK + lane * VEC);
            vj[j] = to_f32(vh[row0 + rr + j]);
            if (MODE == 3) {
#pragma unroll
                for (int e = 0; e < VEC; ++e) s[j].x[e] *= av[e];
            }
        }
        float sq[ROWS], sk[ROWS];
#pragma unroll
        for (int j = 0; j < ROWS; ++j) {
            sq[j] = 0.f;
            sk[j] = 0.f;
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                sq[j] = fmaf(s[j].x[e], qv[e], sq[j]);
                if (kDelta) sk[j] = fmaf(s[j].x[e], kv[e], sk[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < ROWS; ++j) {
            if (kDelta) sk[j] = warp_sum(sk[j]);
        }
#pragma unroll
        for (int j = 0; j < ROWS; ++j) {
            float w;  // coefficient of k in the row update
            if (kDelta) w = b * (vj[j] - a * sk[j]);
            else w = vj[j];
#pragma unroll
            for (int e = 0; e < VEC; ++e) s[j].x[e] = fmaf(w, kv[e], a * s[j].x[e]);
            s[j].store(S + (size_t)(row0 + rr + j) * DK + lane * VEC);
            const float sqr = warp_sum(sq[j]);
            if (lane == 0) o_s[row0 + rr + j] = (MODE == 0) ? (sqr + w * kq) * inv_den
                                                            : fmaf(a, sqr, w * kq);
        }
    }
    __syncthreads();
    for (int t = threadIdx.x; t < DV; t += kDecodeThreads) o[nh * DV + t] = from_f32<IO>(o_s[t]);
}

template <int MODE, typename IO>
cudaError_t launch_mode(const DecodeArgs &a) {
    const dim3 grid((unsigned)((size_t)a.N * a.H));
    const IO *q = static_cast<const IO *>(a.q);
    const IO *k = static_cast<const IO *>(a.k);
    const IO *v = static_cast<const IO *>(a.v);
    IO *o = static_cast<IO *>(a.o);
#define LA_DECODE_CASE(DKc, DVc)                                                            \
    if (a.dk == DKc && a.dv == DVc) {                                                       \
        timer_begin(a.stream);                                                              \
        decode_kernel<MODE, DKc, DVc, IO><<<grid, kDecodeThreads, 0, a.stream>>>(            \
            q, k, v, a.gate, a.beta, a.state, a.z, o, a.gate_heads);                        \
        timer_end(a.stream);                                                                \
        note_launches(1);                                                                   \
        return cudaGetLastError();                                                          \
    }
    LA_DECODE_CASE(128, 128)
    LA_DECODE_CASE(64, 64)
    LA_DECODE_CASE(128, 64)
    LA_DECODE_CASE(64, 128)
#undef LA_DECODE_CASE
    return cudaErrorInvalidValue;
}

template <typename IO>
cudaError_t launch_io(const DecodeArgs &a) {
    switch (a.mode) {
        case LA_MODE_ELU1_NORM: return launch_mode<0, IO>(a);
        case LA_MODE_GATED: return launch_mode<1, IO>(a);
        case LA_MODE_GATED_DELTA: return launch_mode<2, IO>(a);
        case LA_MODE_KDA: return launch_mode<3, IO>(a);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a) {
    return a.dtype == LA_BF16 ? launch_io<__nv_bfloat16>(a) : launch_io<float>(a);
}

}  // namespace la

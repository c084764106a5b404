// varlen.cu -- support kernel for packed variable-length sequences (la_prefill_varlen).
//
// The tensor-core kernels return at once for a sequence with no tokens, leaving its
// state slot as it was.  Without an initial state that slot must read S_0 = 0 (and
// z_0 = 0): this kernel writes those zeros, one CTA per (sequence, head).
#include "la_internal.cuh"

namespace la {
namespace {

__global__ void __launch_bounds__(256)
zero_empty_kernel(int H, int T, int dk, int dv, const int *__restrict__ cu, float *__restrict__ state,
                  float *__restrict__ z) {
    const int sq = blockIdx.x / H;
    const int a = cu[sq], b = cu[sq + 1];
    const int tb = min(max(a, 0), T), te = min(max(b, tb), T);   // the kernels' clamping
    if (te > tb) return;
    float4 *s = reinterpret_cast<float4 *>(state + (size_t)blockIdx.x * dv * dk);
    for (int i = threadIdx.x; i < dv * dk / 4; i += blockDim.x) s[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (z)
        for (int i = threadIdx.x; i < dk; i += blockDim.x) z[(size_t)blockIdx.x * dk + i] = 0.f;
}

}  // namespace

cudaError_t launch_zero_empty_sequences(const PrefillArgs &a) {
    timer_begin(a.stream);
    zero_empty_kernel<<<(unsigned)((size_t)a.nseq * a.H), 256, 0, a.stream>>>(a.H, a.T, a.dk, a.dv, a.cu,
                                                                              a.state, a.z);
    timer_end(a.stream);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace la

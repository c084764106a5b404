// la_internal.cuh -- declarations shared by the translation units of liblinattn.
// Nothing here is part of the public ABI (include/la.h).
#pragma once

#include <cstdint>
#include <initializer_list>
#include <utility>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/la.h"

namespace la {

// Device-side failure word.  A kernel whose bounded wait runs out ORs a code into it
// and returns early; la_check_status() reads and clears it.  Kernels receive its
// address as an argument (device_error_word()), so no relocatable device code is needed.
enum : unsigned { kErrTimeout = 1u, kErrBadLaunch = 2u, kErrBadInput = 4u };
unsigned *device_error_word();   // address on the current device, or nullptr on error

// Counts kernels enqueued by the library (la_kernel_launches()).
void note_launches(unsigned n);

// Optional per-launch device timing (la_launch_timing()): every kernel launch is
// bracketed by timer_begin / timer_end on its stream; each entry point calls
// timer_reset() first.  All three do nothing while timing is disabled.
void timer_reset();
void timer_begin(cudaStream_t s);
void timer_end(cudaStream_t s);

struct PrefillArgs {
    int mode;           // la_mode_t
    int dtype;          // la_dtype_t
    int B, H, T, dk, dv;
    const void *q, *k, *v;
    const float *gate, *beta;
    float *state, *z;
    void *o;
    int chunk;          // resolved (non-zero) chunk size
    bool init_state;
    cudaStream_t stream;
    // Packed variable-length sequences: nullptr for dense [B, H, T, d] tensors.
    // Otherwise B = 1, T = total tokens, the tensors are [H, T, d] (gate/beta [H, T]),
    // sequence s takes tokens [cu[s], cu[s+1]) and owns state slot s of [nseq, H, ..].
    const int *cu = nullptr;
    int nseq = 0;
    // Constant gates (the RetNet decay): gate holds one value per head, [H], used for
    // every token (0: per-token gates).
    int gate_heads = 0;
};

struct DecodeArgs {
    int mode, dtype;
    int N, H, dk, dv;
    const void *q, *k, *v;
    const float *gate, *beta;
    float *state, *z;
    void *o;
    cudaStream_t stream;
    int gate_heads = 0;   // as in PrefillArgs
};

struct ConvArgs {
    int dtype;
    int B, T, H, d, width;   // B: batch rows (prefill) or sequences N (step)
    bool step;               // one token per sequence, window updated in place (win_out)
    bool silu, l2norm;
    const void *x;
    const float *w;
    const void *win_in;      // prefill: nullable (zeros)
    void *win_out;           // prefill: nullable; step: the window, in/out
    void *y;
    cudaStream_t stream;
    // packed variable-length sequences (prefill only): B = N sequences, T = total tokens,
    // x [T, H*d], y [H, T, d], windows [N, W-1, H*d]; nullptr for dense
    const int *cu = nullptr;
};

// Launchers return cudaSuccess or the launch error.  They assume validated arguments.
cudaError_t launch_decode(const DecodeArgs &a);
cudaError_t launch_prefill_simt(const PrefillArgs &a);
bool prefill_simt_supports(int dtype, int dk, int dv, int chunk, int *resolved_chunk);
bool prefill_tc_supports(int mode, int dtype, int dk, int dv, int chunk);
// Workspace of the fastest segment plan, or (minimal) of the smallest segmented plan; the
// launcher picks the fastest plan that fits the workspace it is given.
size_t prefill_tc_workspace_bytes(int mode, int B, int H, int T, bool minimal = false);
cudaError_t launch_prefill_tc(const PrefillArgs &a, void *workspace, size_t workspace_bytes);
// The single-pass gated-delta prefill (d_v split over four CTAs per head, no workspace):
// whether it serves a call of BH head rows (dense or packed), and its launcher.
bool prefill_gdn_selected(int mode, int BH, bool packed);
cudaError_t launch_prefill_gdn(const PrefillArgs &a, void *workspace, size_t workspace_bytes);
// la_prefill_conv: the short convolution of q, k, v fused into the gated-delta prefill's
// first pass (dense, bf16, d = 128; the workspace of the two-pass variant is required).
struct ConvSpec {
    const void *x[3];      // [B, T, H*128] token-major q, k, v projections
    const float *w[3];     // [H*128, width] taps
    const void *win_in;    // [3, B, width-1, H*128] or nullptr
    void *win_out;         // [3, B, width-1, H*128] or nullptr; never overlaps win_in
    void *y;               // [3, B, H, T, 128] out: the convolved q, k, v
    int width;
    unsigned fqk, fv;      // LA_CONV_* flags for q and k, for v
};
cudaError_t launch_prefill_gdn_conv(const PrefillArgs &a, const ConvSpec &cs, void *workspace,
                                    size_t workspace_bytes);
// Workspace with which it runs its two-pass variant (per-chunk factors formed in parallel).
size_t prefill_gdn_workspace_bytes(int BH, int T);
// KDA (mode 3) on the same chain kernel, two-pass only: whether a call of BH head rows
// qualifies, the workspace it needs (its per-chunk records), and its launcher (which also
// needs a 16-byte aligned gate tensor).
bool prefill_kda2_selected(int mode, int BH, bool packed);
size_t prefill_kda2_workspace_bytes(int BH, int T);
cudaError_t launch_prefill_kda2(const PrefillArgs &a, void *workspace, size_t workspace_bytes);
cudaError_t launch_short_conv(const ConvArgs &a);
// Workspace of la_prefill_backward_delta (0 for other modes).
size_t delta_backward_workspace_bytes(int mode, int B, int H, int T, int d_k, int d_v);
// Zero the state (and z) of every packed sequence with no tokens (cu[s+1] <= cu[s]).
cudaError_t launch_zero_empty_sequences(const PrefillArgs &a);

// True if the byte ranges [p, p + n) and [q, q + m) share a byte.
inline bool overlap(const void *p, size_t n, const void *q, size_t m) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(q);
    return p && q && n && m && a < b + m && b < a + n;
}

using Span = std::pair<const void *, size_t>;

// True if the buffers a call writes share no byte with one another or with any buffer it
// only reads (null spans are skipped).  The kernels read inputs while they write outputs,
// so an overlap would be a race, not an in-place update.
inline bool writes_disjoint(std::initializer_list<Span> writes, std::initializer_list<Span> reads) {
    for (auto w = writes.begin(); w != writes.end(); ++w) {
        for (auto u = w + 1; u != writes.end(); ++u)
            if (overlap(w->first, w->second, u->first, u->second)) return false;
        for (const Span &r : reads)
            if (overlap(w->first, w->second, r.first, r.second)) return false;
    }
    return true;
}

// fp32 <-> I/O element helpers used by the CUDA-core kernels.
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// phi(x) = elu(x) + 1 (the lesson's feature map), in fp32.
__device__ __forceinline__ float feature_phi(float x) { return x > 0.f ? x + 1.f : expf(x); }

}  // namespace la

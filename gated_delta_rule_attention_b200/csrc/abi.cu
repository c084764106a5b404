// abi.cu -- the extern "C" boundary of liblinattn (declared in include/la.h).
//
// Host-side only: argument validation, chunk resolution, dispatch to a kernel launcher
// on the caller's stream, and the device failure word.  No entry point allocates
// device memory or keeps a pointer past its return.
#include "la_internal.cuh"

#include <atomic>
#include <cstdint>
#include <initializer_list>
#include <mutex>
#include <utility>

namespace la {

static std::atomic<unsigned long long> g_launches{0};
void note_launches(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

__device__ unsigned g_device_error;

unsigned *device_error_word() {
    constexpr int kMaxDevices = 64;
    static unsigned *addr[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        addr[dev] = static_cast<unsigned *>(p);
    }
    return addr[dev];
}

namespace {

constexpr long long kMaxElems = 1ll << 40;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// True if `p` is memory the current device can address as global memory.
bool device_pointer(const void *p) {
    if (!p) return false;
    cudaPointerAttributes attr;
    const cudaError_t err = cudaPointerGetAttributes(&attr, p);
    if (err != cudaSuccess) {
        (void)cudaGetLastError();  // clear the non-sticky error this query may leave
        return false;
    }
    if (attr.type == cudaMemoryTypeManaged) return true;
    if (attr.type != cudaMemoryTypeDevice) return false;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    return attr.device == dev;
}

bool tensor_ok(const void *p, uintptr_t align) { return p && aligned(p, align) && device_pointer(p); }

la_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? LA_OK : LA_ERR_CUDA; }

// Modes that take beta (the delta rule).
bool delta_mode(int mode) { return mode == LA_MODE_GATED_DELTA || mode == LA_MODE_KDA; }
// The RetNet mode is the scalar-gate mode with one constant gate per head.
int internal_mode(int mode) { return mode == LA_MODE_RETNET ? (int)LA_MODE_GATED : mode; }

bool dims_ok(int dk, int dv) { return (dk == 64 || dk == 128) && (dv == 64 || dv == 128); }

// Bytes of a call's gate tensor: per token (a scalar, or d_k values in the per-channel mode)
// or one value per head (the constant-decay mode).
size_t gate_bytes(int mode, long long tokens_x_heads, int H, int d_k) {
    if (mode == LA_MODE_RETNET) return sizeof(float) * (size_t)H;
    return sizeof(float) * (size_t)tokens_x_heads * (mode == LA_MODE_KDA ? d_k : 1);
}

}  // namespace
}  // namespace la

using namespace la;

extern "C" la_status_t la_prefill(la_mode_t mode, la_dtype_t dtype, int B, int H, int T, int d_k,
                                  int d_v, const void *q, const void *k, const void *v,
                                  const float *gate, const float *beta, float *state, float *z,
                                  void *o, int chunk, unsigned flags, void *workspace,
                                  size_t workspace_bytes, void *stream) {
    timer_reset();
    if (mode < LA_MODE_ELU1_NORM || mode > LA_MODE_RETNET) return LA_ERR_INVALID_ARG;
    if (mode == LA_MODE_RETNET && !tensor_ok(gate, 4)) return LA_ERR_INVALID_ARG;
    if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || T < 0) return LA_ERR_INVALID_ARG;
    if (flags & ~LA_FLAG_INIT_STATE) return LA_ERR_INVALID_ARG;
    if (chunk < 0) return LA_ERR_INVALID_ARG;
    if (!dims_ok(d_k, d_v)) return LA_ERR_UNSUPPORTED;
    const long long BH = (long long)B * H;
    if (BH > INT32_MAX || BH * T * (long long)(d_k > d_v ? d_k : d_v) > kMaxElems)
        return LA_ERR_INVALID_ARG;
    const bool init = (flags & LA_FLAG_INIT_STATE) != 0;
    if (!tensor_ok(state, 16)) return LA_ERR_INVALID_ARG;
    if (mode == LA_MODE_ELU1_NORM && !tensor_ok(z, 16)) return LA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (init) return LA_OK;
        cudaError_t e = cudaMemsetAsync(state, 0, sizeof(float) * BH * d_v * d_k, st);
        if (e == cudaSuccess && mode == LA_MODE_ELU1_NORM)
            e = cudaMemsetAsync(z, 0, sizeof(float) * BH * d_k, st);
        return from_cuda(e);
    }
    if (!tensor_ok(q, 16) || !tensor_ok(k, 16) || !tensor_ok(v, 16) || !tensor_ok(o, 16))
        return LA_ERR_INVALID_ARG;
    if (mode != LA_MODE_ELU1_NORM && gate && !tensor_ok(gate, 4)) return LA_ERR_INVALID_ARG;
    if (delta_mode(mode) && !tensor_ok(beta, 4)) return LA_ERR_INVALID_ARG;
    {
        const size_t es = dtype == LA_BF16 ? 2 : 4, th = (size_t)BH * T;
        const bool z_used = mode == LA_MODE_ELU1_NORM;
        if (!writes_disjoint({{o, th * d_v * es}, {state, sizeof(float) * BH * d_v * d_k},
                              {z_used ? z : nullptr, sizeof(float) * BH * d_k}},
                             {{q, th * d_k * es}, {k, th * d_k * es}, {v, th * d_v * es},
                              {z_used ? nullptr : gate, gate_bytes(mode, (long long)th, H, d_k)},
                              {delta_mode(mode) ? beta : nullptr, sizeof(float) * th},
                              {workspace, workspace ? workspace_bytes : 0}}))
            return LA_ERR_INVALID_ARG;
    }

    PrefillArgs a;
    a.mode = internal_mode(mode);
    a.gate_heads = (mode == LA_MODE_RETNET) ? H : 0;
    a.dtype = dtype;
    a.B = B; a.H = H; a.T = T; a.dk = d_k; a.dv = d_v;
    a.q = q; a.k = k; a.v = v;
    a.gate = (mode == LA_MODE_ELU1_NORM) ? nullptr : gate;
    a.beta = delta_mode(mode) ? beta : nullptr;
    a.state = state;
    a.z = (mode == LA_MODE_ELU1_NORM) ? z : nullptr;
    a.o = o;
    a.init_state = init;
    a.stream = st;
    if (workspace && workspace_bytes && !tensor_ok(workspace, 16)) return LA_ERR_INVALID_ARG;
    if (prefill_tc_supports(internal_mode(mode), dtype, d_k, d_v, chunk)) {
        a.chunk = 64;
        return from_cuda(launch_prefill_tc(a, workspace, workspace ? workspace_bytes : 0));
    }
    int resolved = 0;
    if (!prefill_simt_supports(dtype, d_k, d_v, chunk, &resolved)) return LA_ERR_UNSUPPORTED;
    a.chunk = resolved;
    return from_cuda(launch_prefill_simt(a));
}

extern "C" la_status_t la_prefill_varlen(la_mode_t mode, la_dtype_t dtype, int N, int H, int T,
                                         int d_k, int d_v, const int *cu_seqlens, const void *q,
                                         const void *k, const void *v, const float *gate,
                                         const float *beta, float *state, float *z, void *o,
                                         int chunk, unsigned flags, void *stream) {
    timer_reset();
    if (mode < LA_MODE_ELU1_NORM || mode > LA_MODE_RETNET) return LA_ERR_INVALID_ARG;
    if (mode == LA_MODE_RETNET && !tensor_ok(gate, 4)) return LA_ERR_INVALID_ARG;
    if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    if (N < 1 || H < 1 || T < 0) return LA_ERR_INVALID_ARG;
    if (flags & ~LA_FLAG_INIT_STATE) return LA_ERR_INVALID_ARG;
    if (chunk < 0) return LA_ERR_INVALID_ARG;
    if (!dims_ok(d_k, d_v)) return LA_ERR_UNSUPPORTED;
    if ((long long)N * H > INT32_MAX || (long long)H * T * (d_k > d_v ? d_k : d_v) > kMaxElems)
        return LA_ERR_INVALID_ARG;
    const bool init = (flags & LA_FLAG_INIT_STATE) != 0;
    if (!tensor_ok(cu_seqlens, 4) || !tensor_ok(state, 16)) return LA_ERR_INVALID_ARG;
    if (mode == LA_MODE_ELU1_NORM && !tensor_ok(z, 16)) return LA_ERR_INVALID_ARG;
    if (T > 0) {
        if (!tensor_ok(q, 16) || !tensor_ok(k, 16) || !tensor_ok(v, 16) || !tensor_ok(o, 16))
            return LA_ERR_INVALID_ARG;
        if (mode != LA_MODE_ELU1_NORM && gate && !tensor_ok(gate, 4)) return LA_ERR_INVALID_ARG;
        if (delta_mode(mode) && !tensor_ok(beta, 4)) return LA_ERR_INVALID_ARG;
    }
    {
        const size_t es = dtype == LA_BF16 ? 2 : 4, th = (size_t)H * T;
        const bool z_used = mode == LA_MODE_ELU1_NORM;
        if (!writes_disjoint({{T > 0 ? o : nullptr, th * d_v * es},
                              {state, sizeof(float) * N * H * d_v * d_k},
                              {z_used ? z : nullptr, sizeof(float) * N * H * d_k}},
                             {{cu_seqlens, sizeof(int) * (N + 1)},
                              {T > 0 ? q : nullptr, th * d_k * es}, {T > 0 ? k : nullptr, th * d_k * es},
                              {T > 0 ? v : nullptr, th * d_v * es},
                              {z_used || T == 0 ? nullptr : gate, gate_bytes(mode, (long long)th, H, d_k)},
                              {delta_mode(mode) && T > 0 ? beta : nullptr, sizeof(float) * th}}))
            return LA_ERR_INVALID_ARG;
    }
    PrefillArgs a;
    a.mode = internal_mode(mode);
    a.gate_heads = (mode == LA_MODE_RETNET) ? H : 0;
    a.dtype = dtype;
    a.B = 1; a.H = H; a.T = T; a.dk = d_k; a.dv = d_v;
    a.q = q; a.k = k; a.v = v;
    a.gate = (mode == LA_MODE_ELU1_NORM) ? nullptr : gate;
    a.beta = delta_mode(mode) ? beta : nullptr;
    a.state = state;
    a.z = (mode == LA_MODE_ELU1_NORM) ? z : nullptr;
    a.o = o;
    a.init_state = init;
    a.stream = static_cast<cudaStream_t>(stream);
    a.cu = cu_seqlens;
    a.nseq = N;
    if (T == 0) {   // every sequence is empty
        if (init) return LA_OK;
        return from_cuda(launch_zero_empty_sequences(a));
    }
    if (prefill_tc_supports(internal_mode(mode), dtype, d_k, d_v, chunk)) {
        a.chunk = 64;
        cudaError_t e = launch_prefill_tc(a, nullptr, 0);
        if (e == cudaSuccess && !init) e = launch_zero_empty_sequences(a);
        return from_cuda(e);
    }
    int resolved = 0;
    if (!prefill_simt_supports(dtype, d_k, d_v, chunk, &resolved)) return LA_ERR_UNSUPPORTED;
    a.chunk = resolved;
    return from_cuda(launch_prefill_simt(a));
}

extern "C" size_t la_prefill_workspace_size(la_mode_t mode, la_dtype_t dtype, int B, int H, int T,
                                            int d_k, int d_v, int chunk) {
    if (mode < LA_MODE_ELU1_NORM || mode > LA_MODE_RETNET || B < 1 || H < 1 || T < 1)
        return 0;
    if (!prefill_tc_supports(internal_mode(mode), dtype, d_k, d_v, chunk)) return 0;
    return prefill_tc_workspace_bytes(internal_mode(mode), B, H, T);
}

extern "C" la_status_t la_decode_step(la_mode_t mode, la_dtype_t dtype, int N, int H, int d_k,
                                      int d_v, const void *q, const void *k, const void *v,
                                      const float *gate, const float *beta, float *state,
                                      float *z, void *o, void *stream) {
    timer_reset();
    if (mode < LA_MODE_ELU1_NORM || mode > LA_MODE_RETNET) return LA_ERR_INVALID_ARG;
    if (mode == LA_MODE_RETNET && !tensor_ok(gate, 4)) return LA_ERR_INVALID_ARG;
    if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    if (N < 1 || H < 1) return LA_ERR_INVALID_ARG;
    if (!dims_ok(d_k, d_v)) return LA_ERR_UNSUPPORTED;
    const long long NH = (long long)N * H;
    if (NH > INT32_MAX) return LA_ERR_INVALID_ARG;
    const uintptr_t io_align = dtype == LA_BF16 ? 2 : 4;
    if (!tensor_ok(q, io_align) || !tensor_ok(k, io_align) || !tensor_ok(v, io_align) ||
        !tensor_ok(o, io_align) || !tensor_ok(state, 16))
        return LA_ERR_INVALID_ARG;
    if (mode == LA_MODE_ELU1_NORM && !tensor_ok(z, 16)) return LA_ERR_INVALID_ARG;
    if (mode != LA_MODE_ELU1_NORM && gate && !tensor_ok(gate, 4)) return LA_ERR_INVALID_ARG;
    if (delta_mode(mode) && !tensor_ok(beta, 4)) return LA_ERR_INVALID_ARG;
    {
        const size_t es = dtype == LA_BF16 ? 2 : 4;
        const bool z_used = mode == LA_MODE_ELU1_NORM;
        if (!writes_disjoint({{o, (size_t)NH * d_v * es}, {state, sizeof(float) * NH * d_v * d_k},
                              {z_used ? z : nullptr, sizeof(float) * NH * d_k}},
                             {{q, (size_t)NH * d_k * es}, {k, (size_t)NH * d_k * es},
                              {v, (size_t)NH * d_v * es},
                              {z_used ? nullptr : gate, gate_bytes(mode, NH, H, d_k)},
                              {delta_mode(mode) ? beta : nullptr, sizeof(float) * NH}}))
            return LA_ERR_INVALID_ARG;
    }
    DecodeArgs a;
    a.mode = internal_mode(mode);
    a.gate_heads = (mode == LA_MODE_RETNET) ? H : 0;
    a.dtype = dtype;
    a.N = N; a.H = H; a.dk = d_k; a.dv = d_v;
    a.q = q; a.k = k; a.v = v;
    a.gate = (mode == LA_MODE_ELU1_NORM) ? nullptr : gate;
    a.beta = delta_mode(mode) ? beta : nullptr;
    a.state = state;
    a.z = (mode == LA_MODE_ELU1_NORM) ? z : nullptr;
    a.o = o;
    a.stream = static_cast<cudaStream_t>(stream);
    return from_cuda(launch_decode(a));
}

extern "C" la_status_t la_short_conv(la_dtype_t dtype, int B, int T, int H, int d, int width,
                                     const void *x, const float *w, const void *window_in,
                                     void *window_out, void *y, unsigned flags, void *stream) {
    timer_reset();
    if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    if (B < 1 || T < 0 || H < 1 || width < 1 || width > 4) return LA_ERR_INVALID_ARG;
    if (flags & ~(LA_CONV_SILU | LA_CONV_L2NORM)) return LA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return LA_ERR_UNSUPPORTED;
    const long long C = (long long)H * d;
    if (C > INT32_MAX || (long long)B * T * C > kMaxElems) return LA_ERR_INVALID_ARG;
    if (!tensor_ok(w, 4)) return LA_ERR_INVALID_ARG;
    const size_t es = dtype == LA_BF16 ? 2 : 4;
    const size_t win_bytes = (size_t)B * (width - 1) * C * es;
    const void *win_in = width > 1 ? window_in : nullptr;
    void *win_out = width > 1 ? window_out : nullptr;
    if (win_in && !tensor_ok(win_in, 16)) return LA_ERR_INVALID_ARG;
    if (win_out && !tensor_ok(win_out, 16)) return LA_ERR_INVALID_ARG;
    if (win_in != win_out && overlap(win_in, win_bytes, win_out, win_bytes)) return LA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (!win_out || win_out == win_in) return LA_OK;
        return from_cuda(win_in ? cudaMemcpyAsync(win_out, win_in, win_bytes, cudaMemcpyDeviceToDevice, st)
                                : cudaMemsetAsync(win_out, 0, win_bytes, st));
    }
    if (!tensor_ok(x, 16) || !tensor_ok(y, 16)) return LA_ERR_INVALID_ARG;
    const size_t xy_bytes = (size_t)B * T * C * es;
    if (overlap(x, xy_bytes, y, xy_bytes) || overlap(y, xy_bytes, win_in, win_bytes) ||
        overlap(y, xy_bytes, win_out, win_bytes) || overlap(x, xy_bytes, win_out, win_bytes))
        return LA_ERR_INVALID_ARG;
    ConvArgs a;
    a.dtype = dtype;
    a.B = B; a.T = T; a.H = H; a.d = d; a.width = width;
    a.step = false;
    a.silu = (flags & LA_CONV_SILU) != 0;
    a.l2norm = (flags & LA_CONV_L2NORM) != 0;
    a.x = x; a.w = w; a.win_in = win_in; a.win_out = win_out; a.y = y;
    a.stream = st;
    return from_cuda(launch_short_conv(a));
}

extern "C" la_status_t la_short_conv_varlen(la_dtype_t dtype, int N, int T, int H, int d,
                                            int width, const int *cu_seqlens, const void *x,
                                            const float *w, const void *window_in,
                                            void *window_out, void *y, unsigned flags,
                                            void *stream) {
    timer_reset();
    if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    if (N < 1 || T < 0 || H < 1 || width < 1 || width > 4) return LA_ERR_INVALID_ARG;
    if (flags & ~(LA_CONV_SILU | LA_CONV_L2NORM)) return LA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return LA_ERR_UNSUPPORTED;
    const long long C = (long long)H * d;
    if (C > INT32_MAX || (long long)T * C > kMaxElems || (long long)N * C * width > kMaxElems)
        return LA_ERR_INVALID_ARG;
    if (!tensor_ok(w, 4) || !tensor_ok(cu_seqlens, 4)) return LA_ERR_INVALID_ARG;
    const size_t es = dtype == LA_BF16 ? 2 : 4;
    const size_t win_bytes = (size_t)N * (width - 1) * C * es;
    const void *win_in = width > 1 ? window_in : nullptr;
    void *win_out = width > 1 ? window_out : nullptr;
    if (win_in && !tensor_ok(win_in, 16)) return LA_ERR_INVALID_ARG;
    if (win_out && !tensor_ok(win_out, 16)) return LA_ERR_INVALID_ARG;
    if (win_in != win_out && overlap(win_in, win_bytes, win_out, win_bytes)) return LA_ERR_INVALID_ARG;
    if (T > 0) {
        if (!tensor_ok(x, 16) || !tensor_ok(y, 16)) return LA_ERR_INVALID_ARG;
        const size_t xy_bytes = (size_t)T * C * es;
        if (overlap(x, xy_bytes, y, xy_bytes) || overlap(y, xy_bytes, win_in, win_bytes) ||
            overlap(y, xy_bytes, win_out, win_bytes) || overlap(x, xy_bytes, win_out, win_bytes))
            return LA_ERR_INVALID_ARG;
    }
    ConvArgs a;
    a.dtype = dtype;
    a.B = N; a.T = T; a.H = H; a.d = d; a.width = width;
    a.step = false;
    a.silu = (flags & LA_CONV_SILU) != 0;
    a.l2norm = (flags & LA_CONV_L2NORM) != 0;
    a.x = x; a.w = w; a.win_in = win_in; a.win_out = win_out; a.y = y;
    a.stream = static_cast<cudaStream_t>(stream);
    a.cu = cu_seqlens;
    return from_cuda(launch_short_conv(a));
}

extern "C" la_status_t la_short_conv_step(la_dtype_t dtype, int N, int H, int d, int width,
                                          const void *x, const float *w, void *window, void *y,
                                          unsigned flags, void *stream) {
    timer_reset();
    if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    if (N < 1 || H < 1 || width < 1 || width > 4) return LA_ERR_INVALID_ARG;
    if (flags & ~(LA_CONV_SILU | LA_CONV_L2NORM)) return LA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return LA_ERR_UNSUPPORTED;
    const long long C = (long long)H * d;
    if (C > INT32_MAX || (long long)N * C * width > kMaxElems) return LA_ERR_INVALID_ARG;
    if (!tensor_ok(w, 4) || !tensor_ok(x, 16) || !tensor_ok(y, 16)) return LA_ERR_INVALID_ARG;
    void *win = width > 1 ? window : nullptr;
    if (width > 1 && !tensor_ok(win, 16)) return LA_ERR_INVALID_ARG;
    const size_t es = dtype == LA_BF16 ? 2 : 4;
    const size_t xy_bytes = (size_t)N * C * es, win_bytes = (size_t)N * (width - 1) * C * es;
    if (overlap(x, xy_bytes, y, xy_bytes) || overlap(win, win_bytes, x, xy_bytes) ||
        overlap(win, win_bytes, y, xy_bytes))
        return LA_ERR_INVALID_ARG;
    ConvArgs a;
    a.dtype = dtype;
    a.B = N; a.T = 1; a.H = H; a.d = d; a.width = width;
    a.step = true;
    a.silu = (flags & LA_CONV_SILU) != 0;
    a.l2norm = (flags & LA_CONV_L2NORM) != 0;
    a.x = x; a.w = w; a.win_in = win; a.win_out = win; a.y = y;
    a.stream = static_cast<cudaStream_t>(stream);
    return from_cuda(launch_short_conv(a));
}

extern "C" la_status_t la_check_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return LA_ERR_CUDA;
    unsigned *word = device_error_word();
    if (!word) return LA_ERR_CUDA;
    unsigned host = 0;
    if (cudaMemcpy(&host, word, sizeof(host), cudaMemcpyDeviceToHost) != cudaSuccess)
        return LA_ERR_CUDA;
    if (host == 0) return LA_OK;
    const unsigned zero = 0;
    if (cudaMemcpy(word, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
        return LA_ERR_CUDA;
    if (host & kErrTimeout) return LA_ERR_TIMEOUT;
    if (host & kErrBadInput) return LA_ERR_INVALID_ARG;
    return LA_ERR_CUDA;
}

extern "C" const char *la_status_string(la_status_t s) {
    switch (s) {
        case LA_OK: return "LA_OK: success";
        case LA_ERR_INVALID_ARG: return "LA_ERR_INVALID_ARG: invalid argument (pointer, size, mode or dtype)";
        case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED: no kernel for this combination";
        case LA_ERR_CUDA: return "LA_ERR_CUDA: CUDA runtime error";
        case LA_ERR_TIMEOUT: return "LA_ERR_TIMEOUT: a kernel's bounded wait ran out";
    }
    return "unknown la_status_t";
}

extern "C" int la_version(void) { return 100; }

extern "C" unsigned long long la_kernel_launches(void) {
    return g_launches.load(std::memory_order_relaxed);
}

extern "C" size_t la_prefill_conv_workspace_size(int B, int H, int T) {
    if (B < 1 || H < 1 || T < 1 || (long long)B * H > INT32_MAX) return 0;
    return prefill_gdn_workspace_bytes(B * H, T);
}

extern "C" la_status_t la_prefill_conv(la_dtype_t dtype, int B, int H, int T, int d, int width,
                                       const void *xq, const void *xk, const void *xv, const float *wq,
                                       const float *wk, const float *wv, const void *window_in,
                                       void *window_out, unsigned flags_qk, unsigned flags_v, void *y,
                                       const float *gate, const float *beta, float *state, void *o,
                                       unsigned flags, void *workspace, size_t workspace_bytes,
                                       void *stream) {
    timer_reset();
    if (dtype != LA_BF16) return dtype == LA_F32 ? LA_ERR_UNSUPPORTED : LA_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || T < 1 || width < 1 || width > 4) return LA_ERR_INVALID_ARG;
    if (d != 128) return d == 64 ? LA_ERR_UNSUPPORTED : LA_ERR_INVALID_ARG;
    if ((flags & ~LA_FLAG_INIT_STATE) || ((flags_qk | flags_v) & ~(LA_CONV_SILU | LA_CONV_L2NORM)))
        return LA_ERR_INVALID_ARG;
    const long long BH = (long long)B * H;
    if (BH > INT32_MAX || BH * T * d > kMaxElems) return LA_ERR_INVALID_ARG;
    const void *need16[] = {xq, xk, xv, y, o, state, workspace};
    for (const void *p : need16)
        if (!tensor_ok(p, 16)) return LA_ERR_INVALID_ARG;
    const float *need4[] = {wq, wk, wv, beta};
    for (const float *p : need4)
        if (!tensor_ok(p, 4)) return LA_ERR_INVALID_ARG;
    if (gate && !tensor_ok(gate, 4)) return LA_ERR_INVALID_ARG;
    if (width > 1) {
        if (window_in && !tensor_ok(window_in, 16)) return LA_ERR_INVALID_ARG;
        if (window_out && !tensor_ok(window_out, 16)) return LA_ERR_INVALID_ARG;
    }
    if (workspace_bytes < la_prefill_conv_workspace_size(B, H, T)) return LA_ERR_INVALID_ARG;
    const size_t th = (size_t)BH * T, xb = th * d * 2, win = (size_t)3 * B * (width - 1) * H * d * 2;
    const size_t wb = sizeof(float) * (size_t)H * d * width;
    if (!writes_disjoint({{y, 3 * xb}, {o, xb}, {state, sizeof(float) * BH * d * d},
                          {width > 1 ? window_out : nullptr, win}, {workspace, workspace_bytes}},
                         {{xq, xb}, {xk, xb}, {xv, xb}, {wq, wb}, {wk, wb}, {wv, wb},
                          {width > 1 ? window_in : nullptr, win}, {gate, sizeof(float) * th},
                          {beta, sizeof(float) * th}}))
        return LA_ERR_INVALID_ARG;
    PrefillArgs a;
    a.mode = LA_MODE_GATED_DELTA;
    a.dtype = LA_BF16;
    a.B = B; a.H = H; a.T = T; a.dk = d; a.dv = d;
    const __nv_bfloat16 *yb = static_cast<const __nv_bfloat16 *>(y);
    a.q = yb;
    a.k = yb + th * d;
    a.v = yb + 2 * th * d;
    a.gate = gate;
    a.beta = beta;
    a.state = state;
    a.z = nullptr;
    a.o = o;
    a.chunk = 64;
    a.init_state = (flags & LA_FLAG_INIT_STATE) != 0;
    a.stream = static_cast<cudaStream_t>(stream);
    ConvSpec cs;
    cs.x[0] = xq; cs.x[1] = xk; cs.x[2] = xv;
    cs.w[0] = wq; cs.w[1] = wk; cs.w[2] = wv;
    cs.win_in = width > 1 ? window_in : nullptr;
    cs.win_out = width > 1 ? window_out : nullptr;
    cs.y = y;
    cs.width = width;
    cs.fqk = flags_qk;
    cs.fv = flags_v;
    return from_cuda(launch_prefill_gdn_conv(a, cs, workspace, workspace_bytes));
}

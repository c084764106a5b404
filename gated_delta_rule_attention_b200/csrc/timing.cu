// timing.cu -- optional per-launch device timing (la_launch_timing / la_launch_times).
//
// When enabled, every kernel the library enqueues is bracketed by two CUDA events
// recorded on the caller's stream, so that a caller can read how long each launch of
// its last call took on the device, on the stream the launch ran on.  Off by default.
#include "la_internal.cuh"

#include <mutex>

namespace la {
namespace {

constexpr int kMaxTimed = 16;   // launches recorded per call; later ones are not timed

std::mutex g_mu;
bool g_enabled = false;
int g_device = -1;              // device the events belong to
cudaEvent_t g_ev[2 * kMaxTimed];
int g_n = 0;                    // launches recorded in the current call
bool g_open = false;            // a begin event is waiting for its end

bool ensure_events_locked() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (dev == g_device) return true;
    if (g_device >= 0) {
        cudaSetDevice(g_device);
        for (int i = 0; i < 2 * kMaxTimed; ++i) cudaEventDestroy(g_ev[i]);
        cudaSetDevice(dev);
        g_device = -1;
    }
    for (int i = 0; i < 2 * kMaxTimed; ++i) {
        if (cudaEventCreate(&g_ev[i]) != cudaSuccess) {
            for (int j = 0; j < i; ++j) cudaEventDestroy(g_ev[j]);
            return false;
        }
    }
    g_device = dev;
    return true;
}

}  // namespace

void timer_reset() {
    std::lock_guard<std::mutex> lock(g_mu);
    g_n = 0;
    g_open = false;
}

void timer_begin(cudaStream_t s) {
    std::lock_guard<std::mutex> lock(g_mu);
    g_open = false;
    if (!g_enabled || g_n >= kMaxTimed || !ensure_events_locked()) return;
    g_open = cudaEventRecord(g_ev[2 * g_n], s) == cudaSuccess;
}

void timer_end(cudaStream_t s) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_open) return;
    g_open = false;
    if (cudaEventRecord(g_ev[2 * g_n + 1], s) == cudaSuccess) ++g_n;
}

}  // namespace la

extern "C" {

la_status_t la_launch_timing(int enable) {
    std::lock_guard<std::mutex> lock(la::g_mu);
    la::g_enabled = enable != 0;
    la::g_n = 0;
    la::g_open = false;
    return LA_OK;
}

int la_launch_times(float *ms, int max_n) {
    if (ms == nullptr || max_n < 0) return -1;
    std::lock_guard<std::mutex> lock(la::g_mu);
    if (!la::g_enabled || la::g_n == 0) return 0;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return -1;
    if (cur != la::g_device && cudaSetDevice(la::g_device) != cudaSuccess) return -1;
    int n = la::g_n < max_n ? la::g_n : max_n;
    int out = n;
    if (cudaEventSynchronize(la::g_ev[2 * la::g_n - 1]) != cudaSuccess) out = -1;
    for (int i = 0; i < n && out >= 0; ++i)
        if (cudaEventElapsedTime(&ms[i], la::g_ev[2 * i], la::g_ev[2 * i + 1]) != cudaSuccess) out = -1;
    if (cur != la::g_device) cudaSetDevice(cur);
    return out;
}

}  // extern "C"

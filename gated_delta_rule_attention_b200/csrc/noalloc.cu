// noalloc.cu -- la_prefill_noalloc: la_prefill with a library-owned, statically sized
// scratch buffer, for callers that cannot allocate device memory themselves.
//
// Some callers have no device allocator they may use: code that runs inside another
// framework's memory pool (where a cudaMalloc would bypass the pool's accounting and
// can fail once the pool has reserved the device), or processes that reserve all device
// memory at start-up.  They can still pass inputs and outputs, but not the optional
// segment workspace of la_prefill.  This entry point supplies that workspace from a
// file-scope device array instead, and never calls cudaMalloc, cudaFree or any
// allocating library routine.
//
// The array (kStaticWorkspaceBytes) lives in the library's device image: every GPU that
// loads the library holds it until the process exits.  In host code its name is only a
// host-side stand-in, so its device address is looked up once per device with
// cudaGetSymbolAddress (with that device current) on the first call made there; that
// first call should therefore come before any stream capture on the device.  All calls
// share the one array and it keeps the last call's contents; nothing in it needs to
// start at zero (every value the kernels read is written earlier in the same call).
// Calls whose work overlaps on the GPU (other streams, other threads) race on it.
#include "la_internal.cuh"

#include <mutex>

namespace la {
namespace {

constexpr size_t kStaticWorkspaceBytes = size_t(24) << 20;   // 24 MiB per device
static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

void *static_workspace_address() {
    constexpr int kMaxDevices = 64;
    static void *addr[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess) {
            (void)cudaGetLastError();
            return nullptr;
        }
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace
}  // namespace la

extern "C" la_status_t la_prefill_noalloc(la_mode_t mode, la_dtype_t dtype, int B, int H, int T,
                                          int d_k, int d_v, const void *q, const void *k,
                                          const void *v, const float *gate, const float *beta,
                                          float *state, float *z, void *o, int chunk,
                                          unsigned flags, void *stream) {
    // The launcher runs the fastest segment plan whose workspace fits in the static array,
    // or, when none fits, the single pass that needs none: every problem la_prefill accepts
    // runs here too.  Should the array's address be unavailable, the call runs without it
    // (la_prefill then checks the arguments and picks the single pass).
    void *ws = nullptr;
    if (la_prefill_workspace_size(mode, dtype, B, H, T, d_k, d_v, chunk) > 0)
        ws = la::static_workspace_address();
    return la_prefill(mode, dtype, B, H, T, d_k, d_v, q, k, v, gate, beta, state, z, o, chunk,
                      flags, ws, ws ? la::kStaticWorkspaceBytes : 0, stream);
}

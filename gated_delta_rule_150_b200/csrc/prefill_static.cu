// prefill_static.cu -- gdr_prefill for callers that cannot allocate memory.
//
// gdr_prefill needs a caller-provided workspace.  Some callers cannot get one:
// code running while a CUDA graph is being captured (cudaMalloc is not a
// capturable operation), plugins inside a host framework that owns every
// allocation and exposes no allocator, and latency-critical serving loops
// where an allocation (or a trip into a caching allocator) is not allowed on
// the request path.  This entry point gives them a prefill that allocates
// nothing: its workspace is a fixed array in the library's own device memory.
//
// The array is a file-scope __device__ variable of kStaticBytes bytes.  Every
// GPU that loads this library holds it until the process exits.  Host code
// cannot use the array's name as a device address; the address comes from
// cudaGetSymbolAddress with the device current.  It is looked up again on
// every call whose stream is not capturing (so a context re-created after
// cudaDeviceReset gets the new module's address), and the last address seen
// on that device is used while a stream is being captured, when a lookup
// that might load the module is not allowed.  The first call on a device
// must therefore come before any stream capture.
#include <cstring>
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kStaticBytes = (size_t)GDR_STATIC_WORKSPACE_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_static_workspace[kStaticBytes];

std::mutex g_mutex;
void* g_addr[kMaxDevices] = {};

// Device address of g_static_workspace on the current device (NULL on error).
// `refresh`: look it up now (stream not capturing) instead of using the
// address cached by an earlier call.
void* static_workspace_address(bool refresh, gdr_status* status) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *status = GDR_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    if (refresh || !g_addr[dev]) {
        if (!refresh) {              // capturing, and no earlier call on this device
            *status = GDR_ERR_CUDA;
            return nullptr;
        }
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || !p) {
            *status = GDR_ERR_CUDA;
            return nullptr;
        }
        g_addr[dev] = p;
    }
    *status = GDR_OK;
    return g_addr[dev];
}

// Whether `stream` is being captured into a CUDA graph (errors count as yes,
// so that no lookup is attempted in a state that cannot be queried).
bool capturing(cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return true;
    return cs != cudaStreamCaptureStatusNone;
}

}  // namespace

extern "C" gdr_status gdr_prefill_static_workspace(const gdr_prefill_args* args, void* stream) {
    if (!args) return GDR_ERR_INVALID_ARG;
    const size_t need = gdr_prefill_workspace_size(args->n_seqs, args->n_heads, args->d_k,
                                                   args->d_v, args->total_tokens,
                                                   args->scalar_decay);
    if (need == 0) {
        // bad sizes: let the regular checks name the error
        gdr_prefill_args probe = *args;
        probe.workspace = nullptr;
        probe.workspace_bytes = 0;
        const gdr_status s = gdr_prefill(&probe, stream);
        return s == GDR_OK ? GDR_ERR_INVALID_ARG : s;
    }
    if (need > kStaticBytes) return GDR_ERR_WORKSPACE;   // beyond the fixed maximum
    gdr_status s = GDR_OK;
    void* ws = static_workspace_address(!capturing(static_cast<cudaStream_t>(stream)), &s);
    if (!ws) return s;
    // Everything the kernels read from the workspace is written earlier in the
    // same call (the error word is cleared, g and the chunk records are fully
    // rewritten), so leftovers of the previous call do not matter.
    gdr_prefill_args a = *args;
    a.workspace = ws;
    a.workspace_bytes = kStaticBytes;
    return gdr_prefill(&a, stream);
}

// Word 0 of the array is the prefill's device-side error word (the workspace
// layout puts it at offset 0): one read of it, then the stream is synchronised.
extern "C" gdr_status gdr_prefill_static_status(void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    gdr_status s = GDR_OK;
    void* ws = static_workspace_address(!capturing(st), &s);
    if (!ws) return s;
    uint32_t word = 0;
    if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return GDR_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return GDR_ERR_CUDA;
    return word == 0 ? GDR_OK : GDR_ERR_TIMEOUT;
}

// noalloc.cu -- qmoe_forward_noalloc: the forward with its scratch memory in a
// fixed, library-owned device array instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// operator: a plugin whose host framework owns all device memory and hands it
// only the input and output buffers, or a serving loop that must not allocate
// while it handles a request. For them the scratch lives in one file-scope
// __device__ array of kNoAllocScratchBytes, which every GPU that loads this
// library holds until the process exits.
//
// In host code the array's name is only a host-side stand-in for the symbol,
// not a device address: the device address is looked up once per device with
// cudaGetSymbolAddress while that device is current, on the first call made
// on it, and kept. Every call shares the one array and the array keeps the
// last call's contents: calls whose GPU work overlaps (different streams, or
// a second host thread) race on it, so a caller must serialise them. The
// forward itself clears the only scratch word that must start at zero (its
// device status word) and writes every other scratch byte before reading it.
#include <mutex>

#include "qmoe_internal.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" {

size_t qmoe_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

qmoe_status qmoe_forward_noalloc(const qmoe_handle* h, int64_t T, const void* x, const void* router_logits,
                                 const void* shared_output, void* y, void* stream) {
    if (!h) return QMOE_INVALID_ARGUMENT;
    if (T < 0) return QMOE_INVALID_ARGUMENT;
    const size_t need = qmoe_workspace_size(h, T);
    if (need > kNoAllocScratchBytes) {
        h->last_error = "qmoe_forward_noalloc: " + std::to_string(T) + " tokens need " + std::to_string(need) +
                        " bytes of scratch, above the fixed " + std::to_string(kNoAllocScratchBytes) +
                        "; use qmoe_forward with a caller workspace";
        return QMOE_INVALID_ARGUMENT;
    }
    int dev = -1;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        h->last_error = "qmoe_forward_noalloc: no usable current device";
        return QMOE_CUDA_ERROR;
    }
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_setup_mu);
        if (!g_scratch_addr[dev]) {
            // the address lookup is not a stream operation; under stream
            // capture it may fail or invalidate the capture, so the first call
            // on a device must come before any capture
            cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
            err = cudaStreamIsCapturing((cudaStream_t)stream, &cs);
            if (err != cudaSuccess || cs != cudaStreamCaptureStatusNone) {
                h->last_error =
                    "qmoe_forward_noalloc: the first call on a device looks up the scratch array's address and "
                    "must not run under stream capture; make one call on this device before capturing";
                return QMOE_INVALID_ARGUMENT;
            }
            void* p = nullptr;
            err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
            if (err != cudaSuccess || !p) {
                h->last_error = std::string("qmoe_forward_noalloc: cudaGetSymbolAddress: ") + cudaGetErrorString(err);
                return QMOE_CUDA_ERROR;
            }
            g_scratch_addr[dev] = p;
        }
        scratch = g_scratch_addr[dev];
    }
    return qmoe_forward(h, T, x, router_logits, shared_output, y, scratch, kNoAllocScratchBytes, stream);
}

qmoe_status qmoe_noalloc_read_device_status(const qmoe_handle* h, void* stream) {
    if (!h) return QMOE_INVALID_ARGUMENT;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        h->last_error = "qmoe_noalloc_read_device_status: no usable current device";
        return QMOE_CUDA_ERROR;
    }
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_setup_mu);
        scratch = g_scratch_addr[dev];
    }
    if (!scratch) {
        h->last_error = "qmoe_noalloc_read_device_status: no qmoe_forward_noalloc call has run on this device";
        return QMOE_INVALID_ARGUMENT;
    }
    // the status word sits at the same offset for every T
    return qmoe_read_device_status(h, scratch, stream);
}

}  // extern "C"

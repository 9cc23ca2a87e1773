// lstm_forward_noalloc: the inference forward without a caller-supplied
// workspace.  Its scratch is a file-scope device array of fixed size, so the
// call itself allocates no device memory.
#include <mutex>

#include "../../include/lstm.h"
#include "lstm_internal.h"

namespace lstm {
size_t forward_workspace_prefix(const lstm_desc* desc);   // lstm_abi.cu
bool desc_is_valid(const lstm_desc* desc);                 // lstm_abi.cu
}

namespace {

// The scratch every call shares.  It occupies LSTM_NOALLOC_SCRATCH_BYTES on
// each GPU on which the library's device code is loaded, until the process
// exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LSTM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name only stands for the symbol, so the address is looked up once
// per device (with that device current) and cached.  A cudaDeviceReset
// unloads the module and invalidates the cached address; callers that reset
// a device do not use this entry point on it again in the same process.
void* scratch_on_current_device() {
    static std::mutex mu;
    static void* addr[kMaxDevices] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

extern "C" lstm_status lstm_forward_noalloc(const lstm_desc* desc, const void* x, const void* h0,
                                            const float* c0, const void* const* w_ih,
                                            const void* const* w_hh, const void* const* b_ih,
                                            const void* const* b_hh, void* out, void* h_n, float* c_n,
                                            cudaStream_t stream) {
    if (!lstm::desc_is_valid(desc)) return LSTM_ERR_INVALID_ARG;
    const size_t need = lstm::forward_workspace_prefix(desc);
    if (need == 0) return LSTM_ERR_UNSUPPORTED;   // valid, but no recurrent plan fits the device
    if (need > (size_t)LSTM_NOALLOC_SCRATCH_BYTES) return LSTM_ERR_WORKSPACE;
    void* scratch = scratch_on_current_device();
    if (!scratch) return LSTM_ERR_CUDA;
    // An inference forward touches only the first `need` bytes of its
    // workspace (see forward_workspace_prefix), which fit in the scratch; the
    // size passed is the full query so the usual argument checks apply.  The
    // forward clears its status word and counters at the start of every call.
    return lstm_forward(desc, x, h0, c0, w_ih, w_hh, b_ih, b_hh, out, h_n, c_n, scratch,
                        lstm_workspace_size(desc), nullptr, 0, stream);
}

extern "C" lstm_status lstm_noalloc_query_status(cudaStream_t stream) {
    void* scratch = scratch_on_current_device();
    if (!scratch) return LSTM_ERR_CUDA;
    // the status word is the first int of the scratch, as in any workspace
    return lstm_query_status(scratch, stream);
}

// gdn_extend_static_scratch: EXTEND for callers that cannot allocate device
// memory.
//
// Some callers have no way to call cudaMalloc before a prefill: engine
// plugins whose enqueue step must not allocate because the host framework's
// allocator owns (and may have reserved nearly all of) device memory, code on
// a latency-critical path that cannot afford the device-wide synchronisation
// cudaMalloc / cudaFree may cause, and hosts that hand the layer only its
// input and output buffers.  This entry point runs the same kernels as
// gdn_extend, with the workspace taken from a fixed array that lives in the
// library's own device memory instead of from the caller.
//
// The array is a file-scope __device__ variable: every GPU on which the
// library is loaded holds GDN_EXTEND_STATIC_SCRATCH_BYTES of it until the
// process exits.  Host code cannot use the array's name as a device address
// (in host code it names a host-side stand-in), so the first call on each
// device asks the runtime for the device address with cudaGetSymbolAddress,
// with that device current, and keeps it for later calls.

#include <mutex>

#include "gdn_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_extend_scratch[GDN_EXTEND_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_extend_scratch on the current device (looked up once).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_extend_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" int gdn_extend_static_scratch(const gdn_config_t* cfg, const gdn_params_t* params,
                                         const void* mixed_qkv, const void* a, const void* b,
                                         const int32_t* cu_seqlens, int32_t N, int32_t T,
                                         const int32_t* state_indices, const int32_t* has_initial_state,
                                         void* conv_state, float* ssm_state, int32_t P, void* out,
                                         gdn_stream_t stream) {
    // every host-side check first, so that only a call that will launch kernels touches the shared array
    gdn::LayerDims d;
    bool nothing = false;
    const int rc = gdn::check_extend_args(cfg, params, mixed_qkv, a, b, cu_seqlens, N, T, state_indices,
                                          has_initial_state, conv_state, ssm_state, P, out, &d, &nothing);
    if (rc != GDN_OK) return rc;
    if (nothing) return GDN_OK;
    if (gdn::extend_workspace_bytes(d, N, T, nullptr) > (size_t)GDN_EXTEND_STATIC_SCRATCH_BYTES)
        return GDN_ERR_WORKSPACE;
    void* scratch = nullptr;
    cudaError_t e = scratch_address(&scratch);
    if (e == cudaSuccess)  // the header holds the chunk count and the error word: start from zero
        e = cudaMemsetAsync(scratch, 0, gdn::kHeaderBytes, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return GDN_ERR_CUDA;  // the runtime's cudaGetLastError() holds the cause
    return gdn_extend(cfg, params, mixed_qkv, a, b, cu_seqlens, N, T, state_indices, has_initial_state, conv_state,
                      ssm_state, P, out, scratch, (size_t)GDN_EXTEND_STATIC_SCRATCH_BYTES, stream);
}

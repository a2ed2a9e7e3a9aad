// Forward entry point that allocates nothing: its scratch lives in a fixed-size array in the
// library's own device memory instead of a caller-supplied workspace.
//
// Who needs it: callers that cannot call cudaMalloc at the point where they run attention,
// e.g. a plug-in inside a host application that owns all device memory and hands the plug-in
// no allocator, or a latency-bound serving loop that forbids cudaMalloc / cudaFree after
// start-up because those calls can synchronise the device and stall other streams.  Such a
// caller still provides Q, K, V, the mask and the outputs; only the scratch comes from here.
//
// The array is a file-scope __device__ object, so every context that loads this library's
// kernels holds EOT_STATIC_SCRATCH_BYTES of it until the module is unloaded (normally process
// exit).  In host code its name is only a host-side stand-in: the device address is looked up
// with cudaGetSymbolAddress, in the context that is current, on every call.  The lookup is a
// host-side query that allocates nothing; keeping no cached address means a caller that makes
// its own driver context current, or one that resets the device, always gets the address of the
// array in the context it is using.
#include "kernels.cuh"

namespace eot {
eot_status forward_impl(const eot_problem* p, const void* Q, const void* K, const void* V, const uint8_t* mask,
                        void* O, float* u_tail, float* v_tail, void* ws, cudaStream_t st);
eot_status validate_problem(const eot_problem* p);
}  // namespace eot

namespace {

static __device__ __align__(256) unsigned char g_static_scratch[EOT_STATIC_SCRATCH_BYTES];

// Device address of g_static_scratch in the current context.
eot_status scratch_address(void** out) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || !ptr) return EOT_ERR_CUDA;
    *out = ptr;
    return EOT_OK;
}

}  // namespace

extern "C" eot_status eot_sinkhorn_fwd_static(const eot_problem* p, const void* Q, const void* K, const void* V,
                                              const uint8_t* mask, void* O, float* u_tail, float* v_tail,
                                              void* stream) {
    eot_status s = eot::validate_problem(p);
    if (s != EOT_OK) return s;
    if (int64_t(p->B) * p->H * p->L == 0) return EOT_OK;
    if (!Q || !K || !V || !O || !u_tail || !v_tail) return EOT_ERR_INVALID_ARGUMENT;
    if (eot::ws_layout(*p, false).total > size_t(EOT_STATIC_SCRATCH_BYTES)) return EOT_ERR_WORKSPACE_TOO_SMALL;
    void* ws = nullptr;
    s = scratch_address(&ws);
    if (s != EOT_OK) return s;
    // The status word (the only region read before it is written) is cleared by the first
    // kernel of every forward call.
    return eot::forward_impl(p, Q, K, V, mask, O, u_tail, v_tail, ws, static_cast<cudaStream_t>(stream));
}

extern "C" eot_status eot_static_last_device_status(void* stream) {
    void* ws = nullptr;
    const eot_status s = scratch_address(&ws);
    if (s != EOT_OK) return s;
    return eot_last_device_status(ws, stream);
}

extern "C" size_t eot_static_scratch_bytes(void) { return size_t(EOT_STATIC_SCRATCH_BYTES); }

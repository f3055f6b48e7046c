// bitnet_pack_nm_noalloc: the per-step pack without a caller-supplied workspace.
//
// Some callers cannot allocate device memory at the point where they pack:
// for example an optimizer step that runs inside a fixed memory pool or an
// embedded runtime whose allocator is not reachable from the call site, or a
// host that must not call cudaMalloc on a latency-critical path.  This entry
// point takes the pack's scratch (the exact-sum accumulators and the code
// threshold) from a fixed array that lives in the library's device image.
//
// The array holds kPackWsBytes bytes on every GPU that loads the library,
// until the process exits.  Its size does not depend on the matrix: the
// scratch serves one matrix per call.  The largest matrix accepted is 2^34
// weights (2^32 groups of four), the bound of the pack's group indexing; the
// scratch's 64-bit exponent bins would stay exact well beyond it.
// Every call clears the array before use.  Calls whose kernels overlap on the
// GPU (different streams, or different host threads on the same device) share
// the array and race; serialise them on one stream.
//
// The array's device address is looked up with cudaGetSymbolAddress on the
// first call on a device and kept, together with the identity of the device's
// CUDA context.  A context that was destroyed and re-created (cudaDeviceReset)
// reloads the library's device image at a new address; the next call sees the
// new context and looks the address up again.
#include <mutex>

#include "../../include/bitnet_sparse.h"
#include "common.cuh"
#include "kernels.h"

namespace {

static __device__ __align__(256) uint8_t g_pack_scratch[bitnet::kPackWsBytes];

constexpr int kMaxDevices = 64;
struct ScratchEntry {
    void *ptr;
    unsigned long long ctx_id;
};
ScratchEntry g_scratch[kMaxDevices] = {};
std::mutex g_scratch_mu;

typedef CUresult (*PFN_ctxGetCurrent)(CUcontext *);
typedef CUresult (*PFN_ctxGetId)(CUcontext, unsigned long long *);

// Unique identity of the calling thread's current context (0 when none is
// current or the driver cannot say).  Driver-assigned context ids are never
// reused within a process, unlike context handles.
unsigned long long current_ctx_id() {
    static PFN_ctxGetCurrent get_current = nullptr;
    static PFN_ctxGetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_ctxGetCurrent>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_ctxGetId>(p);
    });
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    unsigned long long id = 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of the scratch array on the current device.  The host-side
// name g_pack_scratch is only a stand-in for the symbol; the address a kernel
// can use comes from cudaGetSymbolAddress, looked up on the first call on a
// device and again whenever that device's context has changed since.
cudaError_t scratch_for_current_device(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchEntry &ent = g_scratch[dev];
    const unsigned long long id = current_ctx_id();
    if (!ent.ptr || id == 0 || id != ent.ctx_id) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_pack_scratch);   // makes the device's primary context current
        if (e != cudaSuccess) return e;
        ent.ptr = p;
        ent.ctx_id = current_ctx_id();
    }
    *out = ent.ptr;
    return cudaSuccess;
}

}  // namespace

extern "C" bitnet_status bitnet_pack_nm_noalloc(const float *W, bitnet_packed_w *out, float eps, uint8_t *mask_bits,
                                                bitnet_stream_t stream) {
    if (out && out->n_out > 0 && out->k > 0 &&
        static_cast<double>(out->n_out) * static_cast<double>(out->k) > 17179869184.0) {   // 2^34
        bitnet::set_last_error("pack_noalloc: n_out * k exceeds 2^34 weights (2^32 groups of 4), the largest matrix "
                               "this entry point packs");
        return BITNET_ERR_UNSUPPORTED;
    }
    void *ws = nullptr;
    const cudaError_t e = scratch_for_current_device(&ws);
    if (e != cudaSuccess) {
        bitnet::set_last_error(cudaGetErrorString(e));
        return BITNET_ERR_CUDA;
    }
    return bitnet_pack_nm(W, out, eps, mask_bits, ws, bitnet::kPackWsBytes, stream);
}

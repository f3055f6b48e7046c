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
// scratch serves one matrix per call.  Its 64-bit per-exponent bins stay exact
// up to 2^40 weights per matrix, which is the maximum this entry point accepts.
// Every call clears the array before use.  Calls whose kernels overlap on the
// GPU (different streams, or different host threads on the same device) share
// the array and race; serialise them on one stream.
#include <mutex>

#include "../../include/bitnet_sparse.h"
#include "common.cuh"
#include "kernels.h"

namespace {

static __device__ __align__(256) uint8_t g_pack_scratch[bitnet::kPackWsBytes];

constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device.  The host-side
// name g_pack_scratch is only a stand-in for the symbol; the address a kernel
// can use comes from cudaGetSymbolAddress, looked up once per device.
cudaError_t scratch_for_current_device(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_pack_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" bitnet_status bitnet_pack_nm_noalloc(const float *W, bitnet_packed_w *out, float eps, uint8_t *mask_bits,
                                                bitnet_stream_t stream) {
    if (out && out->n_out > 0 && out->k > 0 &&
        static_cast<double>(out->n_out) * static_cast<double>(out->k) > 1099511627776.0) {   // 2^40
        bitnet::set_last_error("pack_noalloc: n_out * k exceeds 2^40 weights, the limit of the fixed scratch");
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

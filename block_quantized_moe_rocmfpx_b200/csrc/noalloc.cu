// noalloc.cu -- moe_ffn_forward_static: the MoE FFN entry point for callers
// that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code that runs where allocation
// is forbidden or unavailable (a real-time serving loop with a no-allocation
// rule, a plugin inside a host application that owns the device allocator, an
// embedded runtime with a fixed memory budget).  For them this entry point
// runs the same kernel as moe_ffn_forward but takes its workspace from a
// file-scope device array compiled into the library, so the caller passes only
// the layer handle, inputs, outputs and a stream.
//
// Facts a caller must know:
//  - The array holds RFX_STATIC_WS_BYTES (16 MiB) on every GPU that loads this
//    library, for as long as the process runs.  Calls whose workspace would be
//    larger (see moe_ffn_workspace_bytes) are rejected with RFX_EUNSUPPORTED.
//    T > 8 runs the prefill path (moe_ffn_prefill) in the same array, so it is
//    available only for layers and T whose prefill workspace fits.
//  - Each call looks up the array's device address with cudaGetSymbolAddress
//    (on the current device).  The first lookup on a device loads the
//    library's device code there: make that first call before any stream
//    capture on the device.  Looking the address up on every call keeps it
//    valid after a device reset.
//  - Every call on a device uses the same array, which keeps the previous
//    call's contents.  Each call clears the control words that must start at
//    zero (an asynchronous memset on the given stream) and rewrites the rest.
//    Calls that overlap on the GPU (different streams, or graphs replayed
//    concurrently) race on the array and give wrong results: serialise them.
//  - Device-side error flags are written into the array and are not reported
//    by this entry point; a caller who needs them uses moe_ffn_forward with a
//    workspace of its own.
#include <cuda_runtime.h>

#include <string>

#include "../../include/rfx.h"
#include "moe_decode.h"

int rfx_fail(int code, const std::string& msg);   // rfx_pack.cpp
size_t rfx_moe_ctrl_bytes(const moe_layer* layer, int T);  // api.cu: bytes of the workspace control block

#define RFX_STATIC_WS_BYTES (16u << 20)

// The workspace array.  In host code its name is only a handle for
// cudaGetSymbolAddress, never a device address.
static __device__ __align__(256) unsigned char g_rfx_static_ws[RFX_STATIC_WS_BYTES];

namespace {

// Device address of the array on the current device.
int static_ws_address(void** out) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_rfx_static_ws);
    if (e != cudaSuccess || !ptr)
        return rfx_fail(RFX_ECUDA, std::string("moe_ffn_forward_static: cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    *out = ptr;
    return RFX_OK;
}

}  // namespace

extern "C" int moe_ffn_forward_static(const moe_layer* layer, const void* x, int T, const int32_t* idx,
                                      const float* w, float* y, void* stream) {
    if (!layer) return rfx_fail(RFX_EINVAL, "moe_ffn_forward_static: null layer");
    if (T == 0) return RFX_OK;   // no token columns: nothing to do
    const size_t need = moe_ffn_workspace_bytes(layer, T);
    if (need == 0)
        return rfx_fail(RFX_EUNSUPPORTED, "moe_ffn_forward_static: need 0 <= T <= 65536, and H and I multiples of 256 "
                                          "when T > 8");
    if (need > RFX_STATIC_WS_BYTES)
        return rfx_fail(RFX_EUNSUPPORTED, "moe_ffn_forward_static: this layer and T need " + std::to_string(need) +
                                              " workspace bytes, more than the static " +
                                              std::to_string((size_t)RFX_STATIC_WS_BYTES) + "; use moe_ffn_forward");
    void* ws = nullptr;
    int rc = static_ws_address(&ws);
    if (rc != RFX_OK) return rc;
    // the control words (work counters, grid-barrier counter, error flag) must
    // start at zero; everything after them is rewritten by the kernels
    const size_t ctrl_bytes = rfx_moe_ctrl_bytes(layer, T);
    cudaError_t e = cudaMemsetAsync(ws, 0, ctrl_bytes, (cudaStream_t)stream);
    if (e != cudaSuccess) return rfx_fail(RFX_ECUDA, std::string("moe_ffn_forward_static: ") + cudaGetErrorString(e));
    return moe_ffn_forward(layer, x, T, idx, w, y, ws, RFX_STATIC_WS_BYTES, stream);
}

// tm_noalloc.cu -- tm_route_topk_noalloc: the router and expert-first bucketing without a
// caller workspace.
//
// Some callers cannot hand this library a scratch buffer: a host framework that owns no
// allocator it may call, or a serving loop that reserves all device memory at start-up and
// allows no allocation afterwards.  For them, the routing scratch (per-chunk expert counts
// and the 128-row tile prefix) lives in a fixed array inside the library's device image.
// Every GPU that loads the library holds that array until the process exits; nothing here
// calls cudaMalloc, cudaFree or any allocating routine.  The array serves as the workspace of
// tm_route_topk, so the two entry points run the same kernels.
#include <stdio.h>

#include <mutex>

#include "tm.h"
#include "tm_internal.h"

namespace tml {
namespace {

// The routing scratch shared by every call of tm_route_topk_noalloc on a device (per-chunk expert
// counts, tile prefix and, for the tensor-core router, the split router weights).
static __device__ __align__(256) unsigned char g_route_scratch[TM_NOALLOC_SCRATCH_BYTES];

std::mutex g_setup_mu;
void* g_scratch_addr[64] = {nullptr};   // device address of g_route_scratch, per device
void* g_scratch_ctx[64] = {nullptr};    // the context that address belongs to

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The calling thread's current driver context (NULL if it cannot be read).
void* current_context() {
    static CtxGetCurrentFn fn = nullptr;
    static bool looked = false;
    if (!looked) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
        looked = true;
    }
    CUcontext c = nullptr;
    if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

// Once per device and context, with that device current: the array's device address.  In host
// code the array's name is only a host-side stand-in, so kernels get this address, never the
// name.  The address is looked up again when the device's context has changed (after a device
// reset the module, and with it the array, is loaded anew).
tm_status scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) { note_cuda_error("tm_route_topk_noalloc: cudaGetDevice", e); return TM_ERR_CUDA; }
    if (dev < 0 || dev >= 64) return TM_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_setup_mu);
    void* ctx = current_context();
    if (!g_scratch_addr[dev] || ctx != g_scratch_ctx[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_route_scratch);
        if (e != cudaSuccess || !p) {
            note_cuda_error("tm_route_topk_noalloc: cudaGetSymbolAddress", e == cudaSuccess ? cudaErrorUnknown : e);
            return TM_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
        g_scratch_ctx[dev] = current_context();
    }
    *out = g_scratch_addr[dev];
    return TM_OK;
}

}  // namespace
}  // namespace tml

using namespace tml;

extern "C" tm_status tm_route_topk_noalloc(const void* x, tm_layout layout, const tm_shape* shape,
                                          const void* norm_gain, const tm_moe_w* w, int32_t* topk_idx,
                                          float* topk_gate, float* logit_gap_opt, float* inv_rms,
                                          int32_t* bucket_offsets, int32_t* bucket_rows, int32_t* slot_of,
                                          void* stream) {
    // the same validation as tm_route_topk: shape, weights and layout through the size query
    const size_t need = (shape && w) ? tm_route_workspace_bytes(shape, layout, w) : 0;
    if (need == 0) return TM_ERR_INVALID_ARG;
    auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!x || !al16(x) || !topk_idx || !topk_gate || !bucket_offsets || !bucket_rows || !slot_of)
        return TM_ERR_INVALID_ARG;
    if (norm_gain && !al16(norm_gain)) return TM_ERR_INVALID_ARG;

    if (need > TM_NOALLOC_SCRATCH_BYTES) {
        char msg[160];
        snprintf(msg, sizeof(msg), "tm_route_topk_noalloc: needs %zu bytes of scratch, the fixed limit is %u", need,
                 (unsigned)TM_NOALLOC_SCRATCH_BYTES);
        note_cuda_error(msg, cudaErrorInvalidValue);
        return TM_ERR_WORKSPACE;
    }
    void* base = nullptr;
    tm_status s = scratch_address(&base);
    if (s != TM_OK) return s;
    // The fixed array is the workspace of the ordinary entry point, so both take the same kernels
    // in the same order and give the same bits.  Nothing in it has to start at zero.
    return tm_route_topk(x, layout, shape, norm_gain, w, topk_idx, topk_gate, logit_gap_opt, inv_rms, bucket_offsets,
                         bucket_rows, slot_of, base, TM_NOALLOC_SCRATCH_BYTES, stream);
}

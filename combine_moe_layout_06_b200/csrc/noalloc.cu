// noalloc.cu -- moe_layout_noalloc(): the layout entry point for callers that
// cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc: code running inside a
// stream capture that must not allocate, allocator-free embedded runtimes,
// or plugins whose host framework owns every device allocation and offers
// no scratch hook.  moe_layout() needs a caller-provided workspace for its
// per-chunk histograms; this variant takes that scratch from a fixed-size
// array in the library's own device memory instead, so the caller passes
// only the inputs and the output arrays.
//
// The scratch is a file-scope __device__ array of MOE_LAYOUT_NOALLOC_SCRATCH_BYTES
// bytes.  Every GPU that loads this library holds it until the process exits.
// In host code the array's name is only a host-side stand-in for the symbol,
// not a device address, so every call looks up its device address on the
// current device with cudaGetSymbolAddress (a host-side lookup that enqueues
// nothing).  Looking it up each time, instead of caching it, keeps the
// address right after a device reset reloads the module elsewhere.
#include "capi_internal.h"

namespace {

__device__ __align__(256) unsigned char g_layout_scratch[MOE_LAYOUT_NOALLOC_SCRATCH_BYTES];

// Device address of g_layout_scratch on the current device, or nullptr.
void* scratch_on_current_device() {
    void* p = nullptr;
    return cudaGetSymbolAddress(&p, g_layout_scratch) == cudaSuccess ? p : nullptr;
}

}  // namespace

extern "C" moe_status_t moe_layout_noalloc(const moe_config_t* c, const int32_t* topk_idx,
                                           const moe_layout_t* L, void* stream) {
    moe_status_t st = moe_check_config(c);
    if (st != MOE_OK) return st;
    st = moe::check_layout_ptrs(c, L);
    if (st != MOE_OK) return st;
    if (c->num_tokens > 0 && topk_idx == nullptr) return MOE_ERR_INVALID_ARG;
    const bool nodes = (c->flags & MOE_FLAG_TWO_LEVEL) != 0;
    const size_t need = moe::layout_scratch_bytes(c->num_tokens, c->num_experts, c->num_nodes, nodes);
    if (need > (size_t)MOE_LAYOUT_NOALLOC_SCRATCH_BYTES) return MOE_ERR_INVALID_ARG;
    void* scratch = scratch_on_current_device();
    if (scratch == nullptr) return MOE_ERR_CUDA;
    // Every scratch word the layout reads is written earlier in the same
    // call (each chunk writes its whole histogram column), so nothing left by
    // a previous call is read and no clearing is needed.
    moe::LayoutParams p = moe::layout_params(c, topk_idx, L);
    p.workspace = scratch;
    return moe::launch_layout(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK
                                                                                  : MOE_ERR_CUDA;
}

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
// not a device address, so its device address is looked up with
// cudaGetSymbolAddress once per device (with that device current) on the
// first call made on it, and cached.
#include <mutex>

#include "moe_layout.h"
#include "moe_kernels.h"

namespace {

__device__ __align__(256) unsigned char g_layout_scratch[MOE_LAYOUT_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_layout_scratch on the current device (looked up on
// the first call per device).  Returns nullptr on failure.
void* scratch_on_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_layout_scratch) != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" moe_status_t moe_layout_noalloc(const moe_config_t* c, const int32_t* topk_idx,
                                           const moe_layout_t* L, void* stream) {
    moe_status_t st = moe_check_config(c);
    if (st != MOE_OK) return st;
    const bool nodes = (c->flags & MOE_FLAG_TWO_LEVEL) != 0;
    const size_t need = moe::layout_workspace_bytes(c->num_tokens, c->num_experts, c->num_nodes, nodes);
    if (need > (size_t)MOE_LAYOUT_NOALLOC_SCRATCH_BYTES) return MOE_ERR_INVALID_ARG;
    const bool tokens = c->num_tokens > 0;
    if (L == nullptr || L->expert_counts == nullptr || L->expert_offsets == nullptr ||
        L->rank_offsets == nullptr || (tokens && L->slot == nullptr) || L->error_word == nullptr ||
        (tokens && topk_idx == nullptr))
        return MOE_ERR_INVALID_ARG;
    if (nodes && (L->node_counts == nullptr || L->node_offsets == nullptr ||
                  (tokens && L->node_slot == nullptr)))
        return MOE_ERR_INVALID_ARG;
    void* scratch = scratch_on_current_device();
    if (scratch == nullptr) return MOE_ERR_CUDA;
    // Every scratch word the layout reads is written earlier in the same
    // call (each chunk writes its whole histogram column), so nothing left by
    // a previous call is read and no clearing is needed.
    moe::LayoutParams p;
    p.T = c->num_tokens;
    p.k = c->top_k;
    p.E = c->num_experts;
    p.R = c->num_ranks;
    p.N = c->num_nodes;
    p.nodes = nodes;
    p.cluster = (c->flags & MOE_FLAG_LAYOUT_CLUSTER) != 0;
    p.topk = topk_idx;
    p.expert_counts = L->expert_counts;
    p.expert_offsets = L->expert_offsets;
    p.rank_offsets = L->rank_offsets;
    p.slot = L->slot;
    p.node_counts = L->node_counts;
    p.node_offsets = L->node_offsets;
    p.node_slot = L->node_slot;
    p.node_src = L->node_src;
    p.err = L->error_word;
    p.workspace = scratch;
    return moe::launch_layout(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK
                                                                                  : MOE_ERR_CUDA;
}

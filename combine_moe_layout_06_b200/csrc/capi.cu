// capi.cu -- the C ABI of libmoe_layout.so (declared in include/moe_layout.h):
// host-side validation, then the kernel launchers.  No entry point
// allocates device memory.
#include "capi_internal.h"

namespace {

using moe::check_layout_ptrs;
using moe::CopyEngine;
using moe::layout_params;

constexpr uint32_t kKnownFlags = MOE_FLAG_TWO_LEVEL | MOE_FLAG_COPY_VECTOR | MOE_FLAG_COPY_BULK |
                                 MOE_FLAG_LAYOUT_CLUSTER | MOE_FLAG_LAYOUT_FUSED |
                                 MOE_FLAG_TWO_LEVEL_FUSED | MOE_FLAG_TWO_LEVEL_SPLIT;

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

CopyEngine engine_of(uint32_t flags) {
    if (flags & MOE_FLAG_COPY_VECTOR) return CopyEngine::kVector;
    if (flags & MOE_FLAG_COPY_BULK) return CopyEngine::kBulk;
    return CopyEngine::kAuto;
}

bool two_level(const moe_config_t* c) { return (c->flags & MOE_FLAG_TWO_LEVEL) != 0; }

int64_t staging_rows(const moe_config_t* c) {
    const int32_t m = c->num_nodes < c->top_k ? c->num_nodes : c->top_k;
    return c->num_tokens * (int64_t)m;
}

moe::RowMoveParams move_params(const moe_config_t* c, const moe_layout_t* L) {
    moe::RowMoveParams p;
    p.T = c->num_tokens;
    p.k = c->top_k;
    p.N = c->num_nodes;
    p.ranks_per_node = c->num_ranks / c->num_nodes;
    p.row_bytes = (size_t)c->hidden * 2;
    p.slot = L->slot;
    p.node_slot = L->node_slot;
    p.node_offsets = L->node_offsets;
    p.rank_offsets = L->rank_offsets;
    p.node_src = L->node_src;
    p.err = L->error_word;
    p.engine = engine_of(c->flags);
    return p;
}

moe_status_t check_dispatch_args(const moe_config_t* c, const moe_layout_t* L, const void* x,
                                 const void* recv, const void* node_staging) {
    moe_status_t st = moe_check_config(c);
    if (st != MOE_OK) return st;
    st = check_layout_ptrs(c, L);
    if (st != MOE_OK) return st;
    if (c->num_tokens == 0) return MOE_OK;
    if (x == nullptr || recv == nullptr) return MOE_ERR_INVALID_ARG;
    if (two_level(c) && node_staging == nullptr) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// early: the layout kernels were enqueued right before on this stream by
// this library and x was complete when they started.
moe_status_t dispatch_impl(const moe_config_t* c, const moe_layout_t* L, const void* x, void* recv,
                           void* node_staging, cudaStream_t s, bool early) {
    moe::RowMoveParams p = move_params(c, L);
    p.early_inputs = early;
    if (!two_level(c)) return cuda_status(moe::launch_dispatch_flat(p, x, recv, s));
    const int64_t rows = staging_rows(c);
    if ((c->flags & MOE_FLAG_TWO_LEVEL_SPLIT) == 0 && p.engine != CopyEngine::kVector &&
        moe::bulk_eligible(p.row_bytes, {x, node_staging, recv}) && moe::node_dispatch_eligible(p))
        return cuda_status(moe::launch_node_dispatch_bulk(p, x, node_staging, rows, recv, s));
    cudaError_t e = moe::launch_node_pack(p, x, node_staging, rows, s);
    p.early_inputs = false;  // expansion reads staging written by the pack
    if (e == cudaSuccess) e = moe::launch_node_expand(p, node_staging, rows, recv, s);
    return cuda_status(e);
}

}  // namespace

namespace moe {

moe_status_t check_layout_ptrs(const moe_config_t* c, const moe_layout_t* L) {
    // Per-token arrays may be NULL only when there are no tokens.
    const bool tokens = c->num_tokens > 0;
    if (L == nullptr || L->expert_counts == nullptr || L->expert_offsets == nullptr ||
        L->rank_offsets == nullptr || (tokens && L->slot == nullptr) || L->error_word == nullptr)
        return MOE_ERR_INVALID_ARG;
    const bool nodes = (c->flags & MOE_FLAG_TWO_LEVEL) != 0;
    if (nodes && (L->node_counts == nullptr || L->node_offsets == nullptr ||
                  (tokens && L->node_slot == nullptr)))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

LayoutParams layout_params(const moe_config_t* c, const int32_t* topk_idx, const moe_layout_t* L) {
    LayoutParams p;
    p.T = c->num_tokens;
    p.k = c->top_k;
    p.E = c->num_experts;
    p.R = c->num_ranks;
    p.N = c->num_nodes;
    p.nodes = (c->flags & MOE_FLAG_TWO_LEVEL) != 0;
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
    p.workspace = L->workspace;
    return p;
}

}  // namespace moe

extern "C" {

const char* moe_status_string(moe_status_t s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument";
        case MOE_ERR_EMPTY_RANK:
            return "MOE_ERR_EMPTY_RANK: num_experts < num_ranks leaves a rank with no expert";
        case MOE_ERR_BAD_NODES:
            return "MOE_ERR_BAD_NODES: num_nodes must divide num_ranks (and be <= MOE_MAX_NODES "
                   "for node staging)";
        case MOE_ERR_EXPERT_OOB: return "MOE_ERR_EXPERT_OOB: expert index outside [0, num_experts)";
        case MOE_ERR_DUP_EXPERT: return "MOE_ERR_DUP_EXPERT: a token names the same expert twice";
        case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT: a bounded device wait gave up";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call failed";
        case MOE_ERR_BAD_LAYOUT: return "MOE_ERR_BAD_LAYOUT: a slot outside the receive buffer";
    }
    return "unknown moe_status_t";
}

moe_status_t moe_check_config(const moe_config_t* c) {
    if (c == nullptr) return MOE_ERR_INVALID_ARG;
    if (c->num_tokens < 0 || c->hidden < 1 || c->num_experts < 1 || c->num_ranks < 1 ||
        c->num_nodes < 1 || c->top_k < 1)
        return MOE_ERR_INVALID_ARG;
    if (c->top_k > c->num_experts || c->top_k > MOE_MAX_TOPK) return MOE_ERR_INVALID_ARG;
    if (c->num_experts > MOE_MAX_EXPERTS) return MOE_ERR_INVALID_ARG;
    if ((c->flags & ~kKnownFlags) != 0) return MOE_ERR_INVALID_ARG;
    if ((c->flags & MOE_FLAG_COPY_VECTOR) && (c->flags & MOE_FLAG_COPY_BULK))
        return MOE_ERR_INVALID_ARG;
    if (c->num_tokens * (int64_t)c->top_k >= ((int64_t)1 << 31)) return MOE_ERR_INVALID_ARG;
    if (c->num_experts < c->num_ranks) return MOE_ERR_EMPTY_RANK;
    if (c->num_nodes > c->num_ranks || c->num_ranks % c->num_nodes != 0) return MOE_ERR_BAD_NODES;
    if (two_level(c) && c->num_nodes > MOE_MAX_NODES) return MOE_ERR_BAD_NODES;
    return MOE_OK;
}

moe_status_t moe_expert_partition(int32_t num_experts, int32_t num_ranks,
                                  int32_t* rank_first_expert) {
    if (num_experts < 1 || num_ranks < 1 || rank_first_expert == nullptr) return MOE_ERR_INVALID_ARG;
    if (num_experts < num_ranks) return MOE_ERR_EMPTY_RANK;
    const moe::Partition p = moe::Partition::make(num_experts, num_ranks, 1);
    for (int32_t r = 0; r <= num_ranks; ++r) rank_first_expert[r] = p.first_expert(r);
    return MOE_OK;
}

moe_status_t moe_layout_workspace_bytes(const moe_config_t* c, size_t* bytes) {
    const moe_status_t st = moe_check_config(c);
    if (st != MOE_OK) return st;
    if (bytes == nullptr) return MOE_ERR_INVALID_ARG;
    *bytes = moe::layout_workspace_bytes(c->num_tokens, c->num_experts, c->num_nodes, two_level(c));
    return MOE_OK;
}

moe_status_t moe_node_staging_rows(const moe_config_t* c, int64_t* rows) {
    const moe_status_t st = moe_check_config(c);
    if (st != MOE_OK) return st;
    if (rows == nullptr) return MOE_ERR_INVALID_ARG;
    *rows = staging_rows(c);
    return MOE_OK;
}

moe_status_t moe_layout(const moe_config_t* c, const int32_t* topk_idx, const moe_layout_t* L,
                        void* stream) {
    moe_status_t st = moe_check_config(c);
    if (st != MOE_OK) return st;
    st = check_layout_ptrs(c, L);
    if (st != MOE_OK) return st;
    if (L->workspace == nullptr || (c->num_tokens > 0 && topk_idx == nullptr))
        return MOE_ERR_INVALID_ARG;
    const moe::LayoutParams p = layout_params(c, topk_idx, L);
    return cuda_status(moe::launch_layout(p, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_dispatch(const moe_config_t* c, const moe_layout_t* L, const void* x, void* recv,
                          void* node_staging, void* stream) {
    const moe_status_t st = check_dispatch_args(c, L, x, recv, node_staging);
    if (st != MOE_OK || c->num_tokens == 0) return st;
    return dispatch_impl(c, L, x, recv, node_staging, static_cast<cudaStream_t>(stream), false);
}

moe_status_t moe_layout_dispatch(const moe_config_t* c, const int32_t* topk_idx,
                                 const moe_layout_t* L, const void* x, void* recv,
                                 void* node_staging, void* stream) {
    moe_status_t st = check_dispatch_args(c, L, x, recv, node_staging);
    if (st != MOE_OK) return st;
    const size_t row_bytes = (size_t)c->hidden * 2;
    const bool pair =
        (c->flags & MOE_FLAG_LAYOUT_FUSED) != 0 && !two_level(c) && c->num_tokens > 0 &&
        L->workspace != nullptr && topk_idx != nullptr &&
        moe::bulk_eligible(row_bytes, {x, recv, L->workspace}) &&
        moe::layout_dispatch_fused_eligible(c->num_tokens, c->top_k, c->num_experts, row_bytes);
    if (pair)
        return cuda_status(moe::launch_layout_dispatch_fused(layout_params(c, topk_idx, L), x, recv,
                                                             row_bytes,
                                                             static_cast<cudaStream_t>(stream)));
    st = moe_layout(c, topk_idx, L, stream);
    if (st != MOE_OK || c->num_tokens == 0) return st;
    return dispatch_impl(c, L, x, recv, node_staging, static_cast<cudaStream_t>(stream), true);
}

moe_status_t moe_combine(const moe_config_t* c, const moe_layout_t* L, const void* expert_out,
                         const float* topk_weights, void* y, void* stream) {
    moe_status_t st = moe_check_config(c);
    if (st != MOE_OK) return st;
    st = check_layout_ptrs(c, L);
    if (st != MOE_OK) return st;
    if (c->num_tokens == 0) return MOE_OK;
    if (expert_out == nullptr || topk_weights == nullptr || y == nullptr) return MOE_ERR_INVALID_ARG;
    moe::CombineParams p;
    p.T = c->num_tokens;
    p.k = c->top_k;
    p.row_bytes = (size_t)c->hidden * 2;
    p.slot = L->slot;
    p.w = topk_weights;
    p.err = L->error_word;
    p.engine = engine_of(c->flags);
    return cuda_status(moe::launch_combine(p, expert_out, y, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_get_error(const moe_layout_t* L, void* stream) {
    if (L == nullptr || L->error_word == nullptr) return MOE_ERR_INVALID_ARG;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t bits = 0;
    cudaError_t e = cudaMemcpyAsync(&bits, L->error_word, sizeof bits, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = cudaMemsetAsync(L->error_word, 0, sizeof bits, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    if (bits & moe::kErrExpertOob) return MOE_ERR_EXPERT_OOB;
    if (bits & moe::kErrDupExpert) return MOE_ERR_DUP_EXPERT;
    if (bits & moe::kErrBadLayout) return MOE_ERR_BAD_LAYOUT;
    if (bits & moe::kErrTimeout) return MOE_ERR_TIMEOUT;
    return MOE_OK;
}

moe_status_t moe_dispatch_decoupled(const moe_config_t* c, const moe_layout_t* L, const void* x,
                                    void* send, void* xfer, void* recv, void* stream) {
    moe_status_t st = moe_check_config(c);
    if (st != MOE_OK) return st;
    if (!two_level(c) || c->num_nodes != c->num_ranks) return MOE_ERR_INVALID_ARG;
    st = check_layout_ptrs(c, L);
    if (st != MOE_OK) return st;
    if (c->num_tokens == 0) return MOE_OK;
    if (x == nullptr || send == nullptr || xfer == nullptr || recv == nullptr)
        return MOE_ERR_INVALID_ARG;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const moe::RowMoveParams p = move_params(c, L);
    const int64_t rows = staging_rows(c);
    cudaError_t e = moe::launch_node_pack(p, x, send, rows, s);
    if (e == cudaSuccess)
        e = moe::launch_copy_rows(send, xfer, L->node_offsets + c->num_nodes, rows, p.row_bytes, s);
    if (e == cudaSuccess) e = moe::launch_node_expand(p, xfer, rows, recv, s);
    return cuda_status(e);
}

moe_status_t moe_combine_decoupled(const moe_config_t* c, const moe_layout_t* L,
                                   const void* expert_out, const float* topk_weights, void* send,
                                   void* xfer, void* y, void* stream) {
    moe_status_t st = moe_check_config(c);
    if (st != MOE_OK) return st;
    st = check_layout_ptrs(c, L);
    if (st != MOE_OK) return st;
    if (c->num_tokens == 0) return MOE_OK;
    if (expert_out == nullptr || topk_weights == nullptr || send == nullptr || xfer == nullptr ||
        y == nullptr)
        return MOE_ERR_INVALID_ARG;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const moe::RowMoveParams p = move_params(c, L);
    const int64_t rows = c->num_tokens * (int64_t)c->top_k;
    cudaError_t e = moe::launch_gather_rows(p, expert_out, send, s);
    if (e == cudaSuccess) e = moe::launch_copy_rows(send, xfer, nullptr, rows, p.row_bytes, s);
    if (e == cudaSuccess) {
        moe::CombineParams cp;
        cp.T = c->num_tokens;
        cp.k = c->top_k;
        cp.row_bytes = p.row_bytes;
        cp.slot = nullptr;
        cp.w = topk_weights;
        cp.err = L->error_word;
        cp.engine = engine_of(c->flags);
        e = moe::launch_combine(cp, xfer, y, s);
    }
    return cuda_status(e);
}

moe_status_t moe_dispatch_allgather(const moe_config_t* c, const moe_layout_t* L, const void* x,
                                    void* gathered, void* recv, void* stream) {
    moe_status_t st = moe_check_config(c);
    if (st != MOE_OK) return st;
    if (c->num_ranks > MOE_MAX_NODES) return MOE_ERR_INVALID_ARG;
    st = check_layout_ptrs(c, L);
    if (st != MOE_OK) return st;
    if (c->num_tokens == 0) return MOE_OK;
    if (x == nullptr || gathered == nullptr || recv == nullptr) return MOE_ERR_INVALID_ARG;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    moe::RowMoveParams p = move_params(c, L);
    p.N = c->num_ranks;  // one lane per rank in the all-gather
    cudaError_t e = moe::launch_allgather_rows(p, x, gathered, s);
    if (e == cudaSuccess) e = moe::launch_rank_select(p, gathered, recv, s);
    return cuda_status(e);
}

moe_status_t moe_combine_reducescatter(const moe_config_t* c, const moe_layout_t* L,
                                       const void* expert_out, const float* topk_weights,
                                       float* partial, void* y, void* stream) {
    moe_status_t st = moe_check_config(c);
    if (st != MOE_OK) return st;
    if (c->num_ranks > MOE_MAX_NODES) return MOE_ERR_INVALID_ARG;
    st = check_layout_ptrs(c, L);
    if (st != MOE_OK) return st;
    if (c->num_tokens == 0) return MOE_OK;
    if (expert_out == nullptr || topk_weights == nullptr || partial == nullptr || y == nullptr)
        return MOE_ERR_INVALID_ARG;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    moe::CombineParams p;
    p.T = c->num_tokens;
    p.k = c->top_k;
    p.row_bytes = (size_t)c->hidden * 2;
    p.slot = L->slot;
    p.w = topk_weights;
    p.err = L->error_word;
    p.engine = engine_of(c->flags);
    cudaError_t e = moe::launch_combine_rank_partials(p, c->num_ranks, L->rank_offsets, expert_out,
                                                      partial, s);
    if (e == cudaSuccess) e = moe::launch_reduce_rank_partials(p, c->num_ranks, partial, y, s);
    return cuda_status(e);
}

namespace {

moe_status_t check_ep(const moe_config_t* c, const moe_layout_t* L, const moe_ep_layout_t* ep) {
    moe_status_t st = moe_check_config(c);
    if (st != MOE_OK) return st;
    if (two_level(c) || c->num_ranks > moe::kMaxEpRanks) return MOE_ERR_INVALID_ARG;
    st = check_layout_ptrs(c, L);
    if (st != MOE_OK) return st;
    if (ep == nullptr || ep->expert_offsets == nullptr || ep->rank_offsets == nullptr ||
        (c->num_tokens > 0 && ep->slot == nullptr))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

}  // namespace

moe_status_t moe_ep_receive_rows(int32_t num_experts, int32_t num_ranks, int32_t num_sources,
                                 const int32_t* counts_all, int64_t* rows_out) {
    if (num_experts < 1 || num_ranks < 1 || num_sources < 1 || counts_all == nullptr ||
        rows_out == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (num_experts < num_ranks) return MOE_ERR_EMPTY_RANK;
    const int64_t n = (int64_t)num_sources * num_experts;
    for (int64_t i = 0; i < n; ++i)
        if (counts_all[i] < 0) return MOE_ERR_INVALID_ARG;
    const moe::Partition part = moe::Partition::make(num_experts, num_ranks, 1);
    for (int32_t r = 0; r < num_ranks; ++r) {
        int64_t rows = 0;
        for (int32_t e = part.first_expert(r); e < part.first_expert(r + 1); ++e)
            for (int32_t g = 0; g < num_sources; ++g) rows += counts_all[(int64_t)g * num_experts + e];
        rows_out[r] = rows;
    }
    return MOE_OK;
}

moe_status_t moe_enable_peer_access(int32_t device, int32_t peer_device) {
    int n = 0;
    if (cudaGetDeviceCount(&n) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    if (device < 0 || peer_device < 0 || device >= n || peer_device >= n || device == peer_device)
        return MOE_ERR_INVALID_ARG;
    int can = 0;
    if (cudaDeviceCanAccessPeer(&can, device, peer_device) != cudaSuccess || !can) return MOE_ERR_CUDA;
    int prev = 0;
    if (cudaGetDevice(&prev) != cudaSuccess || cudaSetDevice(device) != cudaSuccess) return MOE_ERR_CUDA;
    cudaError_t e = cudaDeviceEnablePeerAccess(peer_device, 0);
    if (e == cudaErrorPeerAccessAlreadyEnabled) {
        cudaGetLastError();  // an enabled pair is what was asked for
        e = cudaSuccess;
    }
    const cudaError_t back = cudaSetDevice(prev);
    return e == cudaSuccess && back == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_ep_layout(const moe_config_t* c, int32_t g, int32_t G, const int32_t* topk_idx,
                           const int32_t* counts_all, const moe_layout_t* L,
                           const moe_ep_layout_t* ep, void* stream) {
    const moe_status_t st = check_ep(c, L, ep);
    if (st != MOE_OK) return st;
    if (G < 1 || g < 0 || g >= G || counts_all == nullptr || (c->num_tokens > 0 && topk_idx == nullptr))
        return MOE_ERR_INVALID_ARG;
    moe::EpParams p;
    p.T = c->num_tokens;
    p.k = c->top_k;
    p.E = c->num_experts;
    p.R = c->num_ranks;
    p.G = G;
    p.g = g;
    p.topk = topk_idx;
    p.counts_all = counts_all;
    p.local_expert_offsets = L->expert_offsets;
    p.local_slot = L->slot;
    p.expert_offsets = ep->expert_offsets;
    p.rank_offsets = ep->rank_offsets;
    p.slot = ep->slot;
    p.err = L->error_word;
    return cuda_status(moe::launch_ep_layout(p, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_ep_dispatch(const moe_config_t* c, const moe_layout_t* L, const moe_ep_layout_t* ep,
                             const void* x, void* const* recv_bufs, int64_t capacity_rows,
                             void* stream) {
    const moe_status_t st = check_ep(c, L, ep);
    if (st != MOE_OK || c->num_tokens == 0) return st;
    if (x == nullptr || recv_bufs == nullptr || capacity_rows < 0) return MOE_ERR_INVALID_ARG;
    for (int32_t r = 0; r < c->num_ranks; ++r)
        if (recv_bufs[r] == nullptr) return MOE_ERR_INVALID_ARG;
    moe::RowMoveParams p = move_params(c, L);
    p.N = c->num_ranks;  // one lane per rank
    p.slot = ep->slot;
    p.rank_offsets = ep->rank_offsets;
    return cuda_status(moe::launch_ep_dispatch(p, x, recv_bufs, capacity_rows,
                                               static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_ep_combine(const moe_config_t* c, const moe_layout_t* L, const moe_ep_layout_t* ep,
                            const void* const* eo_bufs, int64_t capacity_rows,
                            const float* topk_weights, void* y, void* stream) {
    const moe_status_t st = check_ep(c, L, ep);
    if (st != MOE_OK || c->num_tokens == 0) return st;
    if (eo_bufs == nullptr || topk_weights == nullptr || y == nullptr || capacity_rows < 0)
        return MOE_ERR_INVALID_ARG;
    for (int32_t r = 0; r < c->num_ranks; ++r)
        if (eo_bufs[r] == nullptr) return MOE_ERR_INVALID_ARG;
    moe::CombineParams p;
    p.T = c->num_tokens;
    p.k = c->top_k;
    p.row_bytes = (size_t)c->hidden * 2;
    p.slot = ep->slot;
    p.w = topk_weights;
    p.err = L->error_word;
    p.engine = engine_of(c->flags);
    return cuda_status(moe::launch_ep_combine(p, c->num_ranks, ep->rank_offsets, eo_bufs,
                                              capacity_rows, y, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_quantize_rows_fp8(const void* src, int64_t rows, int32_t hidden, void* q,
                                   float* scale, void* stream) {
    if (rows < 0 || hidden < 1) return MOE_ERR_INVALID_ARG;
    if (rows == 0) return MOE_OK;
    if (src == nullptr || q == nullptr || scale == nullptr) return MOE_ERR_INVALID_ARG;
    if (!moe::fp8_eligible(hidden, {src}, {q})) return MOE_ERR_INVALID_ARG;
    return cuda_status(moe::launch_quantize_fp8(src, rows, hidden, nullptr, 1, rows, q, scale, nullptr,
                                                static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_dispatch_fp8(const moe_config_t* c, const moe_layout_t* L, const void* x,
                              void* recv_q, float* recv_scale, void* stream) {
    moe_status_t st = moe_check_config(c);
    if (st != MOE_OK) return st;
    if (two_level(c)) return MOE_ERR_INVALID_ARG;
    st = check_layout_ptrs(c, L);
    if (st != MOE_OK) return st;
    if (c->num_tokens == 0) return MOE_OK;
    if (x == nullptr || recv_q == nullptr || recv_scale == nullptr) return MOE_ERR_INVALID_ARG;
    if (!moe::fp8_eligible(c->hidden, {x}, {recv_q})) return MOE_ERR_INVALID_ARG;
    return cuda_status(moe::launch_quantize_fp8(x, c->num_tokens, c->hidden, L->slot, c->top_k,
                                                c->num_tokens * (int64_t)c->top_k, recv_q,
                                                recv_scale, L->error_word,
                                                static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_dispatch_fp8_two_level(const moe_config_t* c, const moe_layout_t* L, const void* x,
                                        void* staging_q, float* staging_scale, void* recv_q,
                                        float* recv_scale, void* stream) {
    moe_status_t st = moe_check_config(c);
    if (st != MOE_OK) return st;
    if (!two_level(c)) return MOE_ERR_INVALID_ARG;
    st = check_layout_ptrs(c, L);
    if (st != MOE_OK) return st;
    if (c->num_tokens == 0) return MOE_OK;
    if (x == nullptr || staging_q == nullptr || staging_scale == nullptr || recv_q == nullptr ||
        recv_scale == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (!moe::fp8_eligible(c->hidden, {x}, {staging_q, recv_q})) return MOE_ERR_INVALID_ARG;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t rows = staging_rows(c);
    if ((c->flags & MOE_FLAG_TWO_LEVEL_SPLIT) == 0) {
        const moe::RowMoveParams p = move_params(c, L);
        if (moe::fp8_node_dispatch_eligible(p, c->hidden, {x, staging_q, recv_q}))
            return cuda_status(moe::launch_fp8_node_dispatch(p, x, c->hidden, staging_q, staging_scale,
                                                             rows, recv_q, recv_scale, s));
    }
    // phase 1: each token quantized once, into the staging row of every node it touches
    cudaError_t e = moe::launch_quantize_fp8(x, c->num_tokens, c->hidden, L->node_slot, c->num_nodes,
                                             rows, staging_q, staging_scale, L->error_word, s,
                                             L->node_offsets);
    // phase 2: the node expansion, once over the codes and once over the scales
    moe::RowMoveParams p = move_params(c, L);
    if (e == cudaSuccess) {
        p.row_bytes = (size_t)c->hidden;
        e = moe::launch_node_expand(p, staging_q, rows, recv_q, s);
    }
    if (e == cudaSuccess) {
        p.row_bytes = sizeof(float);
        e = moe::launch_node_expand(p, staging_scale, rows, recv_scale, s);
    }
    return cuda_status(e);
}

moe_status_t moe_combine_fp8(const moe_config_t* c, const moe_layout_t* L, const void* eo_q,
                             const float* eo_scale, const float* topk_weights, void* y,
                             void* stream) {
    moe_status_t st = moe_check_config(c);
    if (st != MOE_OK) return st;
    st = check_layout_ptrs(c, L);
    if (st != MOE_OK) return st;
    if (c->num_tokens == 0) return MOE_OK;
    if (eo_q == nullptr || eo_scale == nullptr || topk_weights == nullptr || y == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (!moe::fp8_eligible(c->hidden, {y}, {eo_q})) return MOE_ERR_INVALID_ARG;
    moe::CombineParams p;
    p.T = c->num_tokens;
    p.k = c->top_k;
    p.row_bytes = (size_t)c->hidden * 2;
    p.slot = L->slot;
    p.w = topk_weights;
    p.err = L->error_word;
    p.engine = engine_of(c->flags);
    return cuda_status(moe::launch_combine_fp8(p, eo_q, eo_scale, y, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

// dispatch.cu -- fused dispatch and the row-movement kernels around it.
//
// Fused dispatch is the gather-send / scatter-recv of the FUSCO article
// (aigc.bar), section "FUSCO 的核心创新": each token row is read once
// straight from x and written straight into every destination row the
// layout names, so no pack or unpack pass runs.  Two-level dispatch follows
// section "负载均衡与跨节点去重": a row goes once to each node it touches
// (a node staging region, node-major then token order) and is then expanded
// inside the node to that node's expert rows.  The same two kernels with
// one "node" per rank, plus a contiguous copy, form the decoupled
// pack -> copy -> unpack path that section "传统 MoE 通信的痛点" describes.
//
// Register engine: work items are (source row, row chunk) pairs, a chunk
// being 32*VPL vectors, handed out warp by warp over a grid from
// persistent_grid() (resident, or whole resident waves for large
// problems).  Lanes hold the destination rows (k <= 32 slots, or N <= 32
// nodes); the chunk is loaded once with streaming loads and stored to every
// destination with evict-first stores.
#include <climits>
#include <initializer_list>

#include "moe_kernels.h"

namespace moe {

int device_sm_count() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

namespace {

constexpr int kWarpsPerCta = 8;
constexpr int kThreads = kWarpsPerCta * 32;

enum FanMode {
    kFlat = 0, kNodePack = 1, kNodeExpand = 2, kAllGather = 3, kRankSelect = 4, kNodeRows = 5,
    kEpFlat = 6
};

struct FanArgs {
    const void* src;
    void* dst;
    const int* slot;
    const int* node_slot;
    const int* node_offsets;
    const int* rank_offsets;
    const int* node_src;  // [U] staging row -> token (kNodeRows)
    void* ep_bufs[kMaxEpRanks];  // receive buffer of each rank (kEpFlat)
    int64_t ep_capacity;         // rows per receive buffer (kEpFlat)
    int64_t T;
    int k, N, ranks_per_node;
    int64_t row_bytes;
    int64_t rv;        // vectors per row
    int64_t src_rows;  // rows in src (bounds check)
    int64_t dst_rows;  // rows in dst (bounds check)
    int* err;
};

// Flat and node-pack rows are tokens; node-expand rows are (node, token)
// pairs, node-major, so each node's forwarder work is one contiguous run;
// node-rows rows are staging rows, so every warp gets the same number of
// staging rows whatever the nodes' loads (load-aware forwarding).
//
// Where row r's data comes from and goes to: the source row (-1 = nothing to
// move) and, per lane, one destination row (-1 = none).  Computed without
// branching on loaded values, so the loads can be issued a row ahead and
// waited on only when used.
struct RowPlan {
    int64_t src;
    int64_t dst;
    int bad;
};

// Per-lane table, loaded once per warp.  Node-rows mode: lane n < N holds
// node n's first staging row and its receive-row range [lo, hi).  EP mode:
// lane r < N holds rank r's rows [lo, hi) of the concatenated receive
// buffers and the base of its buffer.
struct NodeTable {
    int first;
    int lo, hi;
    unsigned long long buf;
};

__device__ __forceinline__ NodeTable load_ep_table(const FanArgs& a, int lane) {
    NodeTable nt = {INT_MAX, 0, 0, 0ull};
    if (lane < a.N) {
        nt.lo = ld_dep(a.rank_offsets + lane);
        nt.hi = ld_dep(a.rank_offsets + lane + 1);
        nt.buf = reinterpret_cast<unsigned long long>(a.ep_bufs[lane]);
    }
    return nt;
}

__device__ __forceinline__ NodeTable load_node_table(const FanArgs& a, int lane) {
    NodeTable nt;
    nt.buf = 0ull;
    const bool on = lane < a.N;
    nt.first = on ? ld_dep(a.node_offsets + lane) : INT_MAX;
    nt.lo = on ? ld_dep(a.rank_offsets + lane * a.ranks_per_node) : 0;
    nt.hi = on ? ld_dep(a.rank_offsets + (lane + 1) * a.ranks_per_node) : 0;
    return nt;
}

// Node of staging row u: the last node whose first row is <= u (node
// offsets ascend; an empty node shares its first row with the next one).
__device__ __forceinline__ int node_of_row(const NodeTable& nt, int64_t u) {
    return __popc(__ballot_sync(kFullMask, nt.first <= u)) - 1;
}

template <int MODE>
__device__ __forceinline__ RowPlan plan_row(const FanArgs& a, int64_t row, int lane,
                                            const NodeTable& nt) {
    RowPlan p;
    p.dst = -1;
    p.bad = 0;
    if (MODE == kFlat) {
        p.src = row;
        const int s = lane < a.k ? ld_dep(a.slot + row * a.k + lane) : -1;
        const bool ok = s >= 0 && s < a.dst_rows;
        p.dst = ok ? s : -1;
        p.bad = (!ok && s != -1) ? kErrBadLayout : 0;
    } else if (MODE == kNodePack) {
        p.src = row;
        const int ns = lane < a.N ? ld_dep(a.node_slot + row * a.N + lane) : -1;
        const int64_t off = lane < a.N ? (int64_t)ld_dep(a.node_offsets + lane) : 0;
        const int64_t d = off + ns;
        const bool ok = ns >= 0 && d >= 0 && d < a.dst_rows;
        p.dst = ok ? d : -1;
        p.bad = (ns >= 0 && !ok) ? kErrBadLayout : 0;
    } else if (MODE == kAllGather) {
        // every virtual rank (lane r < N) receives a copy of every token
        p.src = row;
        p.dst = lane < a.N ? (int64_t)lane * a.T + row : -1;
    } else if (MODE == kRankSelect) {
        // rank r keeps, from its gathered copy, the token's rows on its experts
        const int r = (int)(row / a.T);
        const int64_t t = row - (int64_t)r * a.T;
        const int lo = ld_dep(a.rank_offsets + r);
        const int hi = ld_dep(a.rank_offsets + r + 1);
        const int s = lane < a.k ? ld_dep(a.slot + t * a.k + lane) : -1;
        p.src = row;
        p.dst = (s >= lo && s < hi && s < a.dst_rows) ? s : -1;
    } else if (MODE == kEpFlat) {
        // the rank whose rows [lo, hi) hold slot s, and the row in its buffer
        const int s = lane < a.k ? ld_dep(a.slot + row * a.k + lane) : -1;
        int r = 0;
        for (int q = 1; q < a.N; ++q) r += s >= __shfl_sync(kFullMask, nt.lo, q) ? 1 : 0;
        const int lo = __shfl_sync(kFullMask, nt.lo, r);
        const int hi = __shfl_sync(kFullMask, nt.hi, r);
        const unsigned long long buf = __shfl_sync(kFullMask, nt.buf, r);
        const int64_t local = (int64_t)s - lo;
        const bool ok = s >= 0 && s < hi && local >= 0 && local < a.ep_capacity && buf != 0ull;
        p.src = row;
        p.dst = ok ? (int64_t)(buf + (unsigned long long)local * (unsigned long long)a.row_bytes) : -1;
        p.bad = (s != -1 && !ok) ? kErrBadLayout : 0;
    } else if (MODE == kNodeRows) {
        // staging row `row` holds token node_src[row] for node n
        const int n = node_of_row(nt, row);
        const int lo = __shfl_sync(kFullMask, nt.lo, n & 31);
        const int hi = __shfl_sync(kFullMask, nt.hi, n & 31);
        const int t = ld_dep(a.node_src + row);  // same for all lanes
        const bool src_ok = n >= 0 && t >= 0 && t < a.T;
        const int s = (src_ok && lane < a.k) ? ld_dep(a.slot + (int64_t)t * a.k + lane) : -1;
        p.src = src_ok ? row : -1;
        p.bad = src_ok ? 0 : kErrBadLayout;
        p.dst = (s >= lo && s < hi && s < a.dst_rows) ? s : -1;
    } else {
        const int n = (int)(row / a.T);
        const int64_t t = row - (int64_t)n * a.T;
        const int ns = ld_dep(a.node_slot + t * a.N + n);  // same for all lanes
        const int64_t srow = (int64_t)ld_dep(a.node_offsets + n) + ns;
        const int lo = ld_dep(a.rank_offsets + n * a.ranks_per_node);
        const int hi = ld_dep(a.rank_offsets + (n + 1) * a.ranks_per_node);
        const int s = lane < a.k ? ld_dep(a.slot + t * a.k + lane) : -1;
        const bool src_ok = ns >= 0 && srow >= 0 && srow < a.src_rows;
        p.src = src_ok ? srow : -1;
        p.bad = (ns >= 0 && !src_ok) ? kErrBadLayout : 0;
        p.dst = (src_ok && s >= lo && s < hi && s < a.dst_rows) ? s : -1;
    }
    return p;
}

// Each warp moves a contiguous, row-major range of (row, chunk) items, so a
// row's plan is loaded once and the next row's plan is fetched while the
// current chunk's loads and stores are in flight.
template <int MODE, typename V, int VPL>
__global__ void __launch_bounds__(kThreads) fanout_kernel(FanArgs a) {
    constexpr int CHUNK = 32 * VPL;
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    int errbits = 0;
    int64_t rows = (MODE == kNodeExpand || MODE == kRankSelect) ? a.T * a.N : a.T;
    NodeTable nt = {INT_MAX, 0, 0, 0ull};
    if (MODE == kEpFlat) nt = load_ep_table(a, lane);
    if (MODE == kNodeRows) {
        // the staging rows the layout filled: node_offsets[N], read here
        nt = load_node_table(a, lane);
        const int64_t U = ld_dep(a.node_offsets + a.N);
        rows = U < 0 ? 0 : (U > a.src_rows ? a.src_rows : U);
        if (rows != U) errbits |= kErrBadLayout;
    }
    const int64_t cpr = (a.rv + CHUNK - 1) / CHUNK;
    const int64_t items = rows * cpr;
    const int64_t nw = (int64_t)gridDim.x * kWarpsPerCta;
    const int64_t gw = (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    const int64_t ib = items * gw / nw, ie = items * (gw + 1) / nw;
    if (ib < ie) {
        int64_t row = ib / cpr;
        int64_t c = ib - row * cpr;
        RowPlan cur = plan_row<MODE>(a, row, lane, nt);
        RowPlan nxt = cur;
        for (int64_t item = ib; item < ie; ++item) {
            const bool last_chunk = c + 1 == cpr;
            if (last_chunk && item + 1 < ie) nxt = plan_row<MODE>(a, row + 1, lane, nt);
            if (cur.src >= 0) {
                const int64_t base = c * CHUNK;
                const V* src = static_cast<const V*>(a.src) + cur.src * a.rv + base;
                V v[VPL];
#pragma unroll
                for (int i = 0; i < VPL; ++i)
                    if (base + i * 32 + lane < a.rv) v[i] = ld_stream(src + i * 32 + lane);
                unsigned m = __ballot_sync(kFullMask, cur.dst >= 0);
                V* dbase = static_cast<V*>(a.dst) + base;
                while (m) {
                    const int j = __ffs(m) - 1;
                    m &= m - 1;
                    const int64_t d = __shfl_sync(kFullMask, cur.dst, j);
                    V* drow = MODE == kEpFlat ? reinterpret_cast<V*>(d) + base : dbase + d * a.rv;
#pragma unroll
                    for (int i = 0; i < VPL; ++i)
                        if (base + i * 32 + lane < a.rv) st_stream(drow + i * 32 + lane, v[i]);
                }
            }
            if (last_chunk) {
                errbits |= cur.bad;
                cur = nxt;
                ++row;
                c = 0;
            } else {
                ++c;
            }
        }
        if (c != 0) errbits |= cur.bad;
    }
    warp_report(a.err, errbits);
}

// dst[t*k + j] = src[slot[t][j]] (decoupled combine's pack).  Items are
// (destination row, row chunk) pairs.
template <typename V, int VPL>
__global__ void __launch_bounds__(kThreads) gather_kernel(FanArgs a) {
    constexpr int CHUNK = 32 * VPL;
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t cpr = (a.rv + CHUNK - 1) / CHUNK;
    const int64_t items = a.T * a.k * cpr;
    const int64_t nw = (int64_t)gridDim.x * kWarpsPerCta;
    const int64_t gw = (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    const int64_t ib = items * gw / nw, ie = items * (gw + 1) / nw;
    int errbits = 0;
    for (int64_t item = ib; item < ie; ++item) {
        const int64_t drow = item / cpr;
        const int64_t base = (item - drow * cpr) * CHUNK;
        const int s = ld_dep(a.slot + drow);   // same for all lanes
        if (s < 0 || s >= a.src_rows) {
            if (s != -1) errbits |= kErrBadLayout;
            continue;
        }
        const V* src = static_cast<const V*>(a.src) + (int64_t)s * a.rv + base;
        V* dst = static_cast<V*>(a.dst) + drow * a.rv + base;
        V v[VPL];
#pragma unroll
        for (int i = 0; i < VPL; ++i)
            if (base + i * 32 + lane < a.rv) v[i] = ld_stream(src + i * 32 + lane);
#pragma unroll
        for (int i = 0; i < VPL; ++i)
            if (base + i * 32 + lane < a.rv) st_stream(dst + i * 32 + lane, v[i]);
    }
    warp_report(a.err, errbits);
}

// Contiguous copy of `rows` rows; the row count may live in device memory
// (the decoupled path's transfer size is known only on the device).
template <typename V>
__global__ void __launch_bounds__(kThreads) copy_kernel(const V* src, V* dst,
                                                        const int* rows_dev, int64_t max_rows,
                                                        int64_t rv) {
    pdl_trigger();
    pdl_wait();
    int64_t rows = max_rows;
    if (rows_dev != nullptr) {
        const int64_t r = ld_dep(rows_dev);
        rows = r < 0 ? 0 : (r < max_rows ? r : max_rows);
    }
    const int64_t n = rows * rv;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (; i + 3 * stride < n; i += 4 * stride) {
        V v0 = ld_stream(src + i), v1 = ld_stream(src + i + stride);
        V v2 = ld_stream(src + i + 2 * stride), v3 = ld_stream(src + i + 3 * stride);
        st_stream(dst + i, v0);
        st_stream(dst + i + stride, v1);
        st_stream(dst + i + 2 * stride, v2);
        st_stream(dst + i + 3 * stride, v3);
    }
    for (; i < n; i += stride) st_stream(dst + i, ld_stream(src + i));
}

// Widest vector that divides the row and every base address.
inline int vec_bytes(size_t row_bytes, std::initializer_list<const void*> ptrs) {
    uintptr_t bits = row_bytes;
    for (const void* p : ptrs) bits |= reinterpret_cast<uintptr_t>(p);
    if (bits % 16 == 0) return 16;
    if (bits % 4 == 0) return 4;
    return 2;
}

template <int MODE, typename V, int VPL>
cudaError_t launch_fan_vpl(FanArgs a, int64_t rows, cudaStream_t stream) {
    constexpr auto kern = fanout_kernel<MODE, V, VPL>;
    const int64_t cpr = (a.rv + 32 * VPL - 1) / (32 * VPL);
    const int grid = persistent_grid<kern>(rows * cpr, kThreads);
    return launch_pdl(kern, dim3(grid), dim3(kThreads), 0, stream, a);
}

// Vectors per lane in one row chunk (compile-time tunable; 4 = 2 KB chunks
// of 16-byte vectors).
#ifndef MOE_DISPATCH_VPL
#define MOE_DISPATCH_VPL 4
#endif

template <int MODE, typename V>
cudaError_t launch_fan_v(FanArgs a, int64_t rows, cudaStream_t stream) {
    constexpr int VPL = MOE_DISPATCH_VPL;
    a.rv /= sizeof(V);
    if (a.rv >= 32 * VPL) return launch_fan_vpl<MODE, V, VPL>(a, rows, stream);
    return launch_fan_vpl<MODE, V, 2>(a, rows, stream);
}

template <int MODE>
cudaError_t launch_fan(FanArgs a, int64_t items, cudaStream_t stream) {
    if (items <= 0) return cudaSuccess;
    switch (vec_bytes((size_t)a.rv, {a.src, a.dst})) {
        case 16: return launch_fan_v<MODE, uint4>(a, items, stream);
        case 4: return launch_fan_v<MODE, uint32_t>(a, items, stream);
        default: return launch_fan_v<MODE, uint16_t>(a, items, stream);
    }
}

FanArgs fan_args(const RowMoveParams& p, const void* src, void* dst, int64_t src_rows,
                 int64_t dst_rows) {
    FanArgs a;
    a.src = src;
    a.dst = dst;
    a.slot = p.slot;
    a.node_slot = p.node_slot;
    a.node_offsets = p.node_offsets;
    a.rank_offsets = p.rank_offsets;
    a.node_src = p.node_src;
    a.T = p.T;
    a.k = p.k;
    a.N = p.N;
    a.ranks_per_node = p.ranks_per_node;
    a.row_bytes = (int64_t)p.row_bytes;
    a.rv = (int64_t)p.row_bytes;  // bytes until the vector width is chosen
    for (int r = 0; r < kMaxEpRanks; ++r) a.ep_bufs[r] = nullptr;
    a.ep_capacity = 0;
    a.src_rows = src_rows;
    a.dst_rows = dst_rows;
    a.err = p.err;
    return a;
}

}  // namespace

// The bulk engine is used unless the register engine is forced or the rows
// are not 16-byte aligned.
inline bool use_bulk(const RowMoveParams& p, std::initializer_list<const void*> ptrs) {
    return p.engine != CopyEngine::kVector && bulk_eligible(p.row_bytes, ptrs);
}

cudaError_t launch_dispatch_flat(const RowMoveParams& p, const void* x, void* recv,
                                 cudaStream_t stream) {
    if (use_bulk(p, {x, recv})) return launch_dispatch_flat_bulk(p, x, recv, stream);
    FanArgs a = fan_args(p, x, recv, p.T, p.T * p.k);
    return launch_fan<kFlat>(a, p.T, stream);
}

cudaError_t launch_node_pack(const RowMoveParams& p, const void* x, void* staging,
                             int64_t staging_rows, cudaStream_t stream) {
    if (use_bulk(p, {x, staging})) return launch_node_pack_bulk(p, x, staging, staging_rows, stream);
    FanArgs a = fan_args(p, x, staging, p.T, staging_rows);
    return launch_fan<kNodePack>(a, p.T, stream);
}

cudaError_t launch_node_expand(const RowMoveParams& p, const void* staging, int64_t staging_rows,
                               void* recv, cudaStream_t stream) {
    if (use_bulk(p, {staging, recv}))
        return launch_node_expand_bulk(p, staging, staging_rows, recv, stream);
    FanArgs a = fan_args(p, staging, recv, staging_rows, p.T * p.k);
    if (p.node_src != nullptr) return launch_fan<kNodeRows>(a, staging_rows, stream);
    return launch_fan<kNodeExpand>(a, p.T * p.N, stream);
}

cudaError_t launch_ep_dispatch(const RowMoveParams& p, const void* x, void* const* bufs,
                               int64_t capacity_rows, cudaStream_t stream) {
    if (p.T <= 0) return cudaSuccess;
    FanArgs a = fan_args(p, x, nullptr, p.T, INT64_MAX);
    uintptr_t bits = (uintptr_t)p.row_bytes | reinterpret_cast<uintptr_t>(x);
    for (int r = 0; r < p.N; ++r) {
        a.ep_bufs[r] = bufs[r];
        bits |= reinterpret_cast<uintptr_t>(bufs[r]);
    }
    a.ep_capacity = capacity_rows;
    if (bits % 16 == 0) return launch_fan_v<kEpFlat, uint4>(a, p.T, stream);
    if (bits % 4 == 0) return launch_fan_v<kEpFlat, uint32_t>(a, p.T, stream);
    return launch_fan_v<kEpFlat, uint16_t>(a, p.T, stream);
}

cudaError_t launch_allgather_rows(const RowMoveParams& p, const void* x, void* gathered,
                                  cudaStream_t stream) {
    // lanes are ranks: N carries the rank count here
    FanArgs a = fan_args(p, x, gathered, p.T, p.T * p.N);
    return launch_fan<kAllGather>(a, p.T, stream);
}

cudaError_t launch_rank_select(const RowMoveParams& p, const void* gathered, void* recv,
                               cudaStream_t stream) {
    FanArgs a = fan_args(p, gathered, recv, p.T * p.N, p.T * p.k);
    return launch_fan<kRankSelect>(a, p.T * p.N, stream);
}

cudaError_t launch_gather_rows(const RowMoveParams& p, const void* src, void* dst,
                               cudaStream_t stream) {
    if (p.T <= 0) return cudaSuccess;
    FanArgs a = fan_args(p, src, dst, p.T * p.k, p.T * p.k);
    const int64_t rows = p.T * p.k;
    switch (vec_bytes(p.row_bytes, {src, dst})) {
        case 16: {
            a.rv /= 16;
            constexpr auto kern = gather_kernel<uint4, 4>;
            const int grid = persistent_grid<kern>(rows * ((a.rv + 127) / 128), kThreads);
            return launch_pdl(kern, dim3(grid), dim3(kThreads), 0, stream, a);
        }
        case 4: {
            a.rv /= 4;
            constexpr auto kern = gather_kernel<uint32_t, 8>;
            const int grid = persistent_grid<kern>(rows * ((a.rv + 255) / 256), kThreads);
            return launch_pdl(kern, dim3(grid), dim3(kThreads), 0, stream, a);
        }
        default: {
            a.rv /= 2;
            constexpr auto kern = gather_kernel<uint16_t, 8>;
            const int grid = persistent_grid<kern>(rows * ((a.rv + 255) / 256), kThreads);
            return launch_pdl(kern, dim3(grid), dim3(kThreads), 0, stream, a);
        }
    }
}

cudaError_t launch_copy_rows(const void* src, void* dst, const int* rows_dev, int64_t max_rows,
                             size_t row_bytes, cudaStream_t stream) {
    if (max_rows <= 0) return cudaSuccess;
    const int grid = device_sm_count() * 8;
    switch (vec_bytes(row_bytes, {src, dst})) {
        case 16:
            return launch_pdl(copy_kernel<uint4>, dim3(grid), dim3(kThreads), 0, stream,
                              static_cast<const uint4*>(src), static_cast<uint4*>(dst), rows_dev,
                              max_rows, (int64_t)(row_bytes / 16));
        case 4:
            return launch_pdl(copy_kernel<uint32_t>, dim3(grid), dim3(kThreads), 0, stream,
                              static_cast<const uint32_t*>(src), static_cast<uint32_t*>(dst),
                              rows_dev, max_rows, (int64_t)(row_bytes / 4));
        default:
            return launch_pdl(copy_kernel<uint16_t>, dim3(grid), dim3(kThreads), 0, stream,
                              static_cast<const uint16_t*>(src), static_cast<uint16_t*>(dst),
                              rows_dev, max_rows, (int64_t)(row_bytes / 2));
    }
}

}  // namespace moe

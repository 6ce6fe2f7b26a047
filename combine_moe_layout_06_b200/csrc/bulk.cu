// bulk.cu -- the bulk-copy (TMA) engine for fused dispatch and combine.
//
// Same operations as the register engine in dispatch.cu / combine.cu
// (FUSCO article, section "FUSCO 的核心创新": rows go straight from where
// they are to where they belong, with no pack or unpack pass), moved by the
// SM's bulk-copy unit instead of by registers:
//
//  dispatch: each warp runs its own pipeline of kDispStages shared-memory
//    stages (12 stages of 2 KB by default, 96 KB per CTA of 4 warps: the best
//    of sweeps over 6-12 stages, 2-4 KB chunks, 2-8 warps and 2-8 items per
//    warp; qwen3 step 204.0 -> 200.8 us against 8 stages).  Lane 0 starts a cp.async.bulk global->shared load of
//    a row chunk into a stage (completion counted on the stage's mbarrier); when
//    it lands, every lane that holds a destination row issues a
//    cp.async.bulk shared->global store of the stage to that row.  Rows are
//    read once and written k times without passing through registers, so
//    store issue no longer throttles the warps.
//
//  combine: each warp's stage holds the chunk of all k expert rows of one
//    token (4 KB: 512-byte chunks for k = 8, one 16-byte vector per lane and
//    row); lanes j < k each start the bulk load of row j, and when the stage
//    lands the warp sums the rows in fp32 from shared memory (same FMA order
//    as the register engine: j = 0 .. k-1 from +0, one RNE store).  Loads
//    for the next stages are in flight while a stage is summed, and small
//    stages leave room for 16 warps per SM to hide the summing latency.
//
// Every mbarrier wait is bounded; a wait that gives up records kErrTimeout,
// stops issuing work, drains what it started and returns.  Every bulk load
// is issued per CTA, into that CTA's own shared memory.  Requires 16-byte
// aligned rows and base addresses.
#include <climits>
#include <cstdlib>
#include <initializer_list>

#include "moe_kernels.h"

namespace moe {
namespace {

// Pipeline shape (compile-time tunables).
#ifndef MOE_BULK_DISP_STAGES
#define MOE_BULK_DISP_STAGES 12
#endif
#ifndef MOE_BULK_DISP_CHUNK
#define MOE_BULK_DISP_CHUNK 2048
#endif
#ifndef MOE_BULK_COMB_STAGES
#define MOE_BULK_COMB_STAGES 3
#endif
#ifndef MOE_BULK_COMB_STAGE_BYTES
#define MOE_BULK_COMB_STAGE_BYTES 4096
#endif
#ifndef MOE_BULK_WARPS
#define MOE_BULK_WARPS 4
#endif
constexpr int kBulkWarps = MOE_BULK_WARPS;
constexpr int kBulkThreads = kBulkWarps * 32;
constexpr int kDispStages = MOE_BULK_DISP_STAGES;
constexpr uint32_t kDispChunk = MOE_BULK_DISP_CHUNK;
constexpr int kCombStages = MOE_BULK_COMB_STAGES;
constexpr uint32_t kCombStageBytes = MOE_BULK_COMB_STAGE_BYTES;  // k row chunks per stage

enum FanMode { kFlat = 0, kNodePack = 1, kNodeExpand = 2, kNodeRows = 3 };

struct BulkArgs {
    const char* src;
    char* dst;
    const float* w;
    const int* slot;          // nullptr (combine): row of (t, j) is t*k + j
    const int* node_slot;
    const int* node_offsets;
    const int* rank_offsets;
    const int* node_src;      // [U] staging row -> token (kNodeRows)
    int64_t T;
    int k, N, ranks_per_node;
    int64_t row_bytes;
    uint32_t chunk;           // bytes per row chunk (multiple of 16)
    int64_t cpr;              // chunks per row
    int64_t src_rows, dst_rows;
    int* err;
    int early;                // start source loads before waiting (see RowMoveParams)
    int late_trigger = 0;     // let the dependent grid launch at the end (pdl_trigger_at_end)
    char* staging = nullptr;  // node_dispatch_kernel: node staging rows
    int64_t staging_rows = 0;
#ifdef MOE_TEST_HOOKS
    // Test builds only: the flat dispatch's warp 0 of block 0 announces the
    // bytes of this item on its stage's mbarrier but issues no load for it,
    // so that wait runs out on a healthy GPU (nothing is left in flight).
    int64_t test_skip_item = -1;
#endif
};

// Drain after a timeout: wait (bounded) for every stage this warp still
// has a load in flight on, then for its bulk stores.
__device__ __forceinline__ void drain(uint64_t* full, uint32_t parity_bits, uint32_t inflight,
                                      int stages) {
    for (int s = 0; s < stages; ++s)
        if (inflight & (1u << s)) (void)mbar_wait(&full[s], (parity_bits >> s) & 1u);
    bulk_wait_all();
}

template <int MODE>
__global__ void __launch_bounds__(kBulkThreads) dispatch_bulk_kernel(BulkArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char* stage0 = smem + (size_t)warp * kDispStages * a.chunk;
    uint64_t* full =
        reinterpret_cast<uint64_t*>(smem + (size_t)kBulkWarps * kDispStages * a.chunk) + warp * kDispStages;
    if (lane == 0) {
        for (int s = 0; s < kDispStages; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    __syncwarp();
    // Flat and node-pack sources are x rows, which need no layout data: with
    // early inputs the first stages are loaded while the layout still runs.
    const bool early = a.early != 0 && (MODE == kFlat || MODE == kNodePack);
    if (!a.late_trigger) pdl_trigger();
    if (!early) pdl_wait();

    int errbits = 0;
    int64_t rows = MODE == kNodeExpand ? a.T * a.N : a.T;
    // node-rows: lane n < N holds node n's first staging row and receive-row
    // range; the rows to move are the node_offsets[N] the layout filled
    int n_first = INT_MAX, n_lo = 0, n_hi = 0;
    if (MODE == kNodeRows) {
        if (lane < a.N) {
            n_first = ld_dep(a.node_offsets + lane);
            n_lo = ld_dep(a.rank_offsets + lane * a.ranks_per_node);
            n_hi = ld_dep(a.rank_offsets + (lane + 1) * a.ranks_per_node);
        }
        const int64_t U = ld_dep(a.node_offsets + a.N);
        rows = U < 0 ? 0 : (U > a.src_rows ? a.src_rows : U);
        if (rows != U) errbits |= kErrBadLayout;
    }
    const int64_t items = rows * a.cpr;
    // a contiguous, row-major range of items per warp
    const int64_t nwarps = (int64_t)gridDim.x * kBulkWarps;
    const int64_t gw = (int64_t)blockIdx.x * kBulkWarps + warp;
    const int64_t first = items * gw / nwarps;
    const int64_t mine = items * (gw + 1) / nwarps - first;

    // Source row of an item (-1: nothing to move), and the chunk geometry.
    auto source = [&](int64_t item, int64_t& row, int64_t& base, uint32_t& bytes) -> int64_t {
        row = item / a.cpr;
        base = (item - row * a.cpr) * (int64_t)a.chunk;
        const int64_t left = a.row_bytes - base;
        bytes = left < (int64_t)a.chunk ? (uint32_t)left : a.chunk;
        if (MODE != kNodeExpand) return row;  // node-rows: the staging row itself
        const int n = (int)(row / a.T);
        const int64_t t = row - (int64_t)n * a.T;
        const int ns = ld_dep(a.node_slot + t * a.N + n);
        if (ns < 0) return -1;
        const int64_t r = (int64_t)ld_dep(a.node_offsets + n) + ns;
        return (r >= 0 && r < a.src_rows) ? r : -2;
    };
    auto issue = [&](int64_t q) {
        const int s = (int)(q % kDispStages);
        int64_t row, base;
        uint32_t bytes;
        const int64_t src_row = source(first + q, row, base, bytes);
#ifdef MOE_TEST_HOOKS
        const bool skip = MODE == kFlat && blockIdx.x == 0 && warp == 0 && first + q == a.test_skip_item;
#else
        constexpr bool skip = false;
#endif
        if (lane == 0) {
            if (src_row >= 0) {
                mbar_arrive_expect_tx(&full[s], bytes);
                if (!skip)
                    bulk_load(stage0 + (size_t)s * a.chunk, a.src + src_row * a.row_bytes + base, bytes,
                              &full[s]);
            } else {
                mbar_arrive_expect_tx(&full[s], 0);  // empty item: complete the phase
            }
        }
    };

    uint32_t parity = 0, inflight = 0;
    for (int64_t q = 0; q < kDispStages && q < mine; ++q) {
        issue(q);
        inflight |= 1u << q;
    }
    if (early) pdl_wait();
    for (int64_t q = 0; q < mine; ++q) {
        const int s = (int)(q % kDispStages);
        const bool ok = __all_sync(kFullMask, mbar_wait(&full[s], (parity >> s) & 1u));
        if (!ok) {
            errbits |= kErrTimeout;
            drain(full, parity, inflight, kDispStages);
            break;
        }
        parity ^= 1u << s;
        inflight &= ~(1u << s);
        int64_t row, base;
        uint32_t bytes;
        const int64_t src_row = source(first + q, row, base, bytes);
        if (src_row == -2) errbits |= kErrBadLayout;
        int64_t dst = -1;
        if (src_row >= 0) {
            if (MODE == kFlat) {
                if (lane < a.k) {
                    const int sl = ld_dep(a.slot + row * a.k + lane);
                    if (sl >= 0 && sl < a.dst_rows) dst = sl;
                    else if (sl != -1) errbits |= kErrBadLayout;
                }
            } else if (MODE == kNodePack) {
                if (lane < a.N) {
                    const int ns = ld_dep(a.node_slot + row * a.N + lane);
                    if (ns >= 0) {
                        const int64_t d = (int64_t)ld_dep(a.node_offsets + lane) + ns;
                        if (d >= 0 && d < a.dst_rows) dst = d;
                        else errbits |= kErrBadLayout;
                    }
                }
            } else if (MODE == kNodeRows) {
                // the node of staging row `row`: the last node starting at or before it
                const int n = __popc(__ballot_sync(kFullMask, n_first <= row)) - 1;
                const int lo = __shfl_sync(kFullMask, n_lo, n & 31);
                const int hi = __shfl_sync(kFullMask, n_hi, n & 31);
                const int t = ld_dep(a.node_src + row);
                if (n < 0 || t < 0 || t >= a.T) {
                    errbits |= kErrBadLayout;
                } else if (lane < a.k) {
                    const int sl = ld_dep(a.slot + (int64_t)t * a.k + lane);
                    if (sl >= lo && sl < hi && sl < a.dst_rows) dst = sl;
                }
            } else {
                const int n = (int)(row / a.T);
                const int64_t t = row - (int64_t)n * a.T;
                const int lo = ld_dep(a.rank_offsets + n * a.ranks_per_node);
                const int hi = ld_dep(a.rank_offsets + (n + 1) * a.ranks_per_node);
                if (lane < a.k) {
                    const int sl = ld_dep(a.slot + t * a.k + lane);
                    if (sl >= lo && sl < hi && sl < a.dst_rows) dst = sl;
                }
            }
        }
        if (dst >= 0) bulk_store(a.dst + dst * a.row_bytes + base, stage0 + (size_t)s * a.chunk, bytes);
        bulk_commit();
        // the stage of item q-1 is free once its stores have read it
        bulk_wait_read<1>();
        __syncwarp();
        if (q >= 1 && q - 1 + kDispStages < mine) {
            issue(q - 1 + kDispStages);
            inflight |= 1u << ((q - 1) % kDispStages);
        }
    }
    if (a.late_trigger) pdl_trigger();
    bulk_wait_all();
    warp_report(a.err, errbits);
}

// Two-level dispatch in one kernel (FUSCO article, section "负载均衡与跨节点
// 去重": a token crosses to a node once, into that node's forwarding region,
// and is fanned out to the node's experts from there).  Per (token, chunk)
// item a warp
//   1. loads the x chunk into a ring of kNfX shared-memory stages (the next
//      kNfX - 1 items' chunks are in flight while this one is handled),
//   2. stores it to the token's staging row of every node it touches (lane
//      31 - n for node n),
//   3. once those stores are complete, reads the staging rows back, up to
//      kNfR nodes at once into read-back buffers, and stores each to the
//      token's receive rows on that node (lane j < k for column j).
// Step 3 reads the staging rows right after they were written, so the reads
// are served by L2 instead of a second pass over HBM.  The staging buffer and
// the receive rows end up exactly as with the two-kernel form (pack, then
// expansion).  Needs N + k <= 32.  Waits are bounded; a wait that gives up
// records kErrTimeout, drains what this warp started and stops.
// Ring shape (compile-time tunables).  4 warps of 6 x stages and 2
// read-back buffers of 2 KB (64 KB per CTA) was the best of a sweep over
// 4-16 warps, 2-8 stages, 1-4 read-back buffers and 1-2 KB chunks on the
// DeepSeek-V3-shaped workload (step 736 us, against 750 us for 8 warps of 2
// stages and 759 us with one read-back buffer).
#ifndef MOE_NF_WARPS
#define MOE_NF_WARPS 4
#endif
#ifndef MOE_NF_XBUFS
#define MOE_NF_XBUFS 6
#endif
#ifndef MOE_NF_IPW
#define MOE_NF_IPW 4
#endif
#ifndef MOE_NF_RBUFS
#define MOE_NF_RBUFS 2
#endif
#ifndef MOE_NF_CHUNK
#define MOE_NF_CHUNK 2048
#endif
constexpr int kNfWarps = MOE_NF_WARPS;
constexpr int kNfThreads = kNfWarps * 32;
constexpr int kNfX = MOE_NF_XBUFS;  // x-chunk ring stages per warp
constexpr int kNfR = MOE_NF_RBUFS;  // staging read-back buffers per warp
constexpr uint32_t kNfChunk = MOE_NF_CHUNK;
static_assert(kNfX >= 2 && kNfX < 31 && kNfR >= 1 && kNfR <= 8, "node dispatch ring shape");
static_assert(kNfChunk % 16 == 0, "bulk copies move multiples of 16 bytes");

__global__ void __launch_bounds__(kNfThreads) node_dispatch_kernel(BulkArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t per_warp = (size_t)(kNfX + kNfR) * a.chunk;
    unsigned char* xbuf = smem + (size_t)warp * per_warp;  // X[kNfX]
    unsigned char* rbuf = xbuf + (size_t)kNfX * a.chunk;    // R[kNfR]
    // bar[s] for s < kNfX: x stage s; bar[kNfX]: the read-back buffers
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + (size_t)kNfWarps * per_warp) + warp * (kNfX + 1);
    constexpr uint32_t kRb = 1u << kNfX;  // parity / in-flight bit of the read-back
    if (lane == 0) {
        for (int i = 0; i <= kNfX; ++i) mbar_init(&bar[i], 1);
        fence_barrier_init();
    }
    __syncwarp();
    const bool early = a.early != 0;
    if (!a.late_trigger) pdl_trigger();
    if (!early) pdl_wait();

    const int64_t items = a.T * a.cpr;
    const int64_t nwarps = (int64_t)gridDim.x * kNfWarps;
    const int64_t gw = (int64_t)blockIdx.x * kNfWarps + warp;
    const int64_t first = items * gw / nwarps;
    const int64_t mine = items * (gw + 1) / nwarps - first;
    auto geometry = [&](int64_t q, int64_t& t, int64_t& off, uint32_t& bytes) {
        const int64_t it = first + q;
        t = it / a.cpr;
        off = (it - t * a.cpr) * (int64_t)a.chunk;
        const int64_t left = a.row_bytes - off;
        bytes = left < (int64_t)a.chunk ? (uint32_t)left : a.chunk;
    };
    auto issue_x = [&](int64_t q) {
        const int b = (int)(q % kNfX);
        int64_t t, off;
        uint32_t bytes;
        geometry(q, t, off, bytes);
        if (lane == 0) {
            mbar_arrive_expect_tx(&bar[b], bytes);
            bulk_load(xbuf + (size_t)b * a.chunk, a.src + t * a.row_bytes + off, bytes, &bar[b]);
        }
    };
    uint32_t parity = 0, inflight = 0;
    for (int64_t q = 0; q < kNfX - 1 && q < mine; ++q) {
        issue_x(q);
        inflight |= 1u << q;
    }
    if (early) pdl_wait();

    // node n: lane n holds its receive-row range [lo, hi); lane 31 - n its
    // first staging row
    const int N = a.N;
    int n_lo = INT_MAX, n_hi = INT_MIN, n_first = 0;
    if (lane < N) {
        n_lo = ld_dep(a.rank_offsets + lane * a.ranks_per_node);
        n_hi = ld_dep(a.rank_offsets + (lane + 1) * a.ranks_per_node);
    }
    const bool stager = lane >= 32 - N;
    const int my_node = 31 - lane;
    if (stager) n_first = ld_dep(a.node_offsets + my_node);

    int errbits = 0;
    int64_t t_cur = -1;
    int sl = -1, nj = -1;
    int64_t srow = -1;
    bool failed = false;
    for (int64_t q = 0; q < mine && !failed; ++q) {
        const int b = (int)(q % kNfX);
        int64_t t, off;
        uint32_t bytes;
        geometry(q, t, off, bytes);
        if (t != t_cur) {
            // column j's receive row and its node; node n's staging row
            sl = -1;
            nj = -1;
            srow = -1;
            if (lane < a.k) {
                const int s = ld_dep(a.slot + t * a.k + lane);
                if (s >= 0 && s < a.dst_rows) sl = s;
                else if (s != -1) errbits |= kErrBadLayout;
            }
            for (int n = 0; n < N; ++n) {
                const int lo = __shfl_sync(kFullMask, n_lo, n);
                const int hi = __shfl_sync(kFullMask, n_hi, n);
                if (sl >= lo && sl < hi) nj = n;
            }
            if (sl >= 0 && nj < 0) errbits |= kErrBadLayout;
            if (stager) {
                const int ns = ld_dep(a.node_slot + t * N + my_node);
                if (ns >= 0) {
                    const int64_t r = (int64_t)n_first + ns;
                    if (r >= 0 && r < a.staging_rows) srow = r;
                    else errbits |= kErrBadLayout;
                }
            }
            t_cur = t;
        }
        if (!__all_sync(kFullMask, mbar_wait(&bar[b], (parity >> b) & 1u))) {
            failed = true;
            break;
        }
        parity ^= 1u << b;
        inflight &= ~(1u << b);
        // 2. one staging row per node touched
        if (srow >= 0) bulk_store(a.staging + srow * a.row_bytes + off, xbuf + (size_t)b * a.chunk, bytes);
        bulk_commit();
        // the previous item's x stage was last read by its staging stores:
        // free once all but the newest group have been read
        bulk_wait_read<1>();
        __syncwarp();
        if (q + kNfX - 1 < mine) {
            issue_x(q + kNfX - 1);
            inflight |= 1u << ((q + kNfX - 1) % kNfX);
        }
        // 3. the staging rows are complete before they are read back
        if (stager) bulk_wait_all();
        __syncwarp();
        unsigned touched = __ballot_sync(kFullMask, srow >= 0);  // bit 31 - n: node n
        while (touched && !failed) {
            // up to kNfR nodes, lowest first, read back together
            int node[kNfR];
            int64_t row_n[kNfR];
            int nb = 0;
#pragma unroll
            for (int i = 0; i < kNfR; ++i) {
                node[i] = -1;
                row_n[i] = 0;
                if (touched) {
                    const int hb = 31 - __clz(touched);
                    touched &= ~(1u << hb);
                    node[i] = 31 - hb;
                    row_n[i] = __shfl_sync(kFullMask, srow, hb);
                    ++nb;
                }
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(&bar[kNfX], bytes * (uint32_t)nb);
#pragma unroll
                for (int i = 0; i < kNfR; ++i)
                    if (i < nb)
                        bulk_load(rbuf + (size_t)i * a.chunk, a.staging + row_n[i] * a.row_bytes + off,
                                  bytes, &bar[kNfX]);
            }
            inflight |= kRb;
            if (!__all_sync(kFullMask, mbar_wait(&bar[kNfX], (parity & kRb) ? 1u : 0u))) {
                failed = true;
                break;
            }
            parity ^= kRb;
            inflight &= ~kRb;
            if (lane < a.k && sl >= 0) {
#pragma unroll
                for (int i = 0; i < kNfR; ++i)
                    if (i < nb && nj == node[i])
                        bulk_store(a.dst + (int64_t)sl * a.row_bytes + off, rbuf + (size_t)i * a.chunk, bytes);
            }
            bulk_commit();
            bulk_wait_read<0>();  // the read-back buffers are free for the next nodes
            __syncwarp();
        }
    }
    if (failed) {
        errbits |= kErrTimeout;
        for (int i = 0; i <= kNfX; ++i)
            if (inflight & (1u << i)) (void)mbar_wait(&bar[i], (parity >> i) & 1u);
    }
    if (a.late_trigger) pdl_trigger();
    bulk_wait_all();
    warp_report(a.err, errbits);
}

__global__ void __launch_bounds__(kBulkThreads) combine_bulk_kernel(BulkArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t stage_bytes = (size_t)a.k * a.chunk;
    unsigned char* stage0 = smem + (size_t)warp * kCombStages * stage_bytes;
    uint64_t* full =
        reinterpret_cast<uint64_t*>(smem + (size_t)kBulkWarps * kCombStages * stage_bytes) + warp * kCombStages;
    if (lane == 0) {
        for (int s = 0; s < kCombStages; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    __syncwarp();
    pdl_trigger();
    pdl_wait();

    const int64_t items = a.T * a.cpr;
    // a contiguous, row-major range of items per warp
    const int64_t nwarps = (int64_t)gridDim.x * kBulkWarps;
    const int64_t gw = (int64_t)blockIdx.x * kBulkWarps + warp;
    const int64_t first = items * gw / nwarps;
    const int64_t mine = items * (gw + 1) / nwarps - first;
    const int64_t eo_rows = a.T * a.k;
    int errbits = 0;

    auto geometry = [&](int64_t item, int64_t& t, int64_t& base, uint32_t& bytes) {
        t = item / a.cpr;
        base = (item - t * a.cpr) * (int64_t)a.chunk;
        const int64_t left = a.row_bytes - base;
        bytes = left < (int64_t)a.chunk ? (uint32_t)left : a.chunk;
    };
    // lane j < k: expert row of (t, j), or -1
    auto row_of = [&](int64_t t) -> int {
        int s = -1;
        if (lane < a.k) {
            s = a.slot ? ld_dep(a.slot + t * a.k + lane) : (int)(t * a.k + lane);
            if (s < 0 || s >= eo_rows) {
                if (s != -1) errbits |= kErrBadLayout;
                s = -1;
            }
        }
        return s;
    };
    auto issue = [&](int64_t q) {
        const int st = (int)(q % kCombStages);
        int64_t t, base;
        uint32_t bytes;
        geometry(first + q, t, base, bytes);
        const int s = row_of(t);
        const unsigned valid = __ballot_sync(kFullMask, s >= 0);
        if (lane == 0) mbar_arrive_expect_tx(&full[st], bytes * (uint32_t)__popc(valid));
        __syncwarp();
        if (s >= 0)
            bulk_load(stage0 + (size_t)st * stage_bytes + (size_t)lane * a.chunk,
                      a.src + (int64_t)s * a.row_bytes + base, bytes, &full[st]);
    };

    uint32_t parity = 0, inflight = 0;
    for (int64_t q = 0; q < kCombStages && q < mine; ++q) {
        issue(q);
        inflight |= 1u << q;
    }
    for (int64_t q = 0; q < mine; ++q) {
        const int st = (int)(q % kCombStages);
        const bool ok = __all_sync(kFullMask, mbar_wait(&full[st], (parity >> st) & 1u));
        if (!ok) {
            errbits |= kErrTimeout;
            drain(full, parity, inflight, kCombStages);
            break;
        }
        parity ^= 1u << st;
        inflight &= ~(1u << st);
        int64_t t, base;
        uint32_t bytes;
        geometry(first + q, t, base, bytes);
        const int s = row_of(t);
        const unsigned valid = __ballot_sync(kFullMask, s >= 0);
        const float wl = lane < a.k ? ld_dep(a.w + t * a.k + lane) : 0.f;
        const unsigned char* stage = stage0 + (size_t)st * stage_bytes;
        char* yrow = a.dst + t * a.row_bytes + base;
        const int nvec = (int)(bytes >> 4);
        // every lane runs every pass (the weight shuffles need the whole warp)
        for (int v0 = 0; v0 < nvec; v0 += 32) {
            const int v = v0 + lane;
            const bool active = v < nvec;
            float acc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = 0.f;
            for (int j = 0; j < a.k; ++j) {
                const float wj = __shfl_sync(kFullMask, wl, j);
                if (!active || !((valid >> j) & 1u)) continue;
                const uint4 x = *reinterpret_cast<const uint4*>(stage + (size_t)j * a.chunk + (size_t)v * 16);
                float f[8];
                unpack_bf16<uint4>(x, f);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = __fmaf_rn(wj, f[e], acc[e]);
            }
            if (active) *reinterpret_cast<uint4*>(yrow + (size_t)v * 16) = pack_bf16<uint4>(acc);
        }
        __syncwarp();
        if (q + kCombStages < mine) {
            if (lane == 0) fence_proxy_async_smem();
            __syncwarp();
            issue(q + kCombStages);
            inflight |= 1u << st;
        }
    }
    warp_report(a.err, errbits);
}

template <auto Kernel>
cudaError_t launch_bulk(BulkArgs a, int64_t items, size_t smem, cudaStream_t stream) {
    if (items <= 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = persistent_grid<Kernel>(items, kBulkThreads, smem);
    a.late_trigger = pdl_trigger_at_end(grid, resident_blocks<Kernel>(kBulkThreads, smem)) ? 1 : 0;
    return launch_pdl(Kernel, dim3(grid), dim3(kBulkThreads), smem, stream, a);
}

BulkArgs bulk_args(const RowMoveParams& p, const void* src, void* dst, int64_t src_rows,
                   int64_t dst_rows, uint32_t chunk) {
    BulkArgs a;
    a.src = static_cast<const char*>(src);
    a.dst = static_cast<char*>(dst);
    a.w = nullptr;
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
    a.chunk = (uint32_t)((int64_t)chunk < a.row_bytes ? chunk : a.row_bytes);
    a.cpr = (a.row_bytes + a.chunk - 1) / a.chunk;
    a.src_rows = src_rows;
    a.dst_rows = dst_rows;
    a.err = p.err;
    a.early = p.early_inputs ? 1 : 0;
    return a;
}

template <int MODE>
cudaError_t launch_disp_bulk(const BulkArgs& a, int64_t rows, cudaStream_t stream) {
    const size_t smem = (size_t)kBulkWarps * kDispStages * (a.chunk + sizeof(uint64_t));
    return launch_bulk<dispatch_bulk_kernel<MODE>>(a, rows * a.cpr, smem, stream);
}

}  // namespace

bool bulk_eligible(size_t row_bytes, std::initializer_list<const void*> ptrs) {
    uintptr_t bits = row_bytes;
    for (const void* p : ptrs) bits |= reinterpret_cast<uintptr_t>(p);
    return row_bytes > 0 && bits % 16 == 0;
}

cudaError_t launch_dispatch_flat_bulk(const RowMoveParams& p, const void* x, void* recv,
                                      cudaStream_t stream) {
    BulkArgs a = bulk_args(p, x, recv, p.T, p.T * p.k, kDispChunk);
#ifdef MOE_TEST_HOOKS
    if (const char* v = std::getenv("MOE_TEST_SKIP_LOAD")) a.test_skip_item = std::atoll(v);
#endif
    return launch_disp_bulk<kFlat>(a, p.T, stream);
}

cudaError_t launch_node_pack_bulk(const RowMoveParams& p, const void* x, void* staging,
                                  int64_t staging_rows, cudaStream_t stream) {
    const BulkArgs a = bulk_args(p, x, staging, p.T, staging_rows, kDispChunk);
    return launch_disp_bulk<kNodePack>(a, p.T, stream);
}

cudaError_t launch_node_expand_bulk(const RowMoveParams& p, const void* staging,
                                    int64_t staging_rows, void* recv, cudaStream_t stream) {
    const BulkArgs a = bulk_args(p, staging, recv, staging_rows, p.T * p.k, kDispChunk);
    if (p.node_src != nullptr) return launch_disp_bulk<kNodeRows>(a, staging_rows, stream);
    return launch_disp_bulk<kNodeExpand>(a, p.T * p.N, stream);
}

bool node_dispatch_eligible(const RowMoveParams& p) { return p.N + p.k <= 32; }

cudaError_t launch_node_dispatch_bulk(const RowMoveParams& p, const void* x, void* staging,
                                      int64_t staging_rows, void* recv, cudaStream_t stream) {
    BulkArgs a = bulk_args(p, x, recv, p.T, p.T * p.k, kNfChunk);
    a.staging = static_cast<char*>(staging);
    a.staging_rows = staging_rows;
    const int64_t items = p.T * a.cpr;
    if (items <= 0) return cudaSuccess;
    const size_t smem = (size_t)kNfWarps * ((kNfX + kNfR) * (size_t)a.chunk + (kNfX + 1) * sizeof(uint64_t));
    cudaError_t e = cudaFuncSetAttribute(node_dispatch_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = persistent_grid<node_dispatch_kernel>(items, kNfThreads, smem, MOE_NF_IPW);
    a.late_trigger =
        pdl_trigger_at_end(grid, resident_blocks<node_dispatch_kernel>(kNfThreads, smem)) ? 1 : 0;
    return launch_pdl(node_dispatch_kernel, dim3(grid), dim3(kNfThreads), smem, stream, a);
}

cudaError_t launch_combine_bulk(const CombineParams& p, const void* expert_out, void* y,
                                cudaStream_t stream) {
    if (p.T <= 0) return cudaSuccess;
    RowMoveParams rp = {};
    rp.T = p.T;
    rp.k = p.k;
    rp.row_bytes = p.row_bytes;
    rp.slot = p.slot;
    rp.err = p.err;
    uint32_t chunk = (kCombStageBytes / (uint32_t)p.k) & ~15u;
    if (chunk < 16) chunk = 16;
    BulkArgs a = bulk_args(rp, expert_out, y, p.T * p.k, p.T, chunk);
    a.w = p.w;
    const size_t smem = (size_t)kBulkWarps * kCombStages * ((size_t)a.k * a.chunk + sizeof(uint64_t));
    return launch_bulk<combine_bulk_kernel>(a, p.T * a.cpr, smem, stream);
}

}  // namespace moe

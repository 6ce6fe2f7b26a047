// layout.cu -- layout ("segment descriptor") kernels.
//
// FUSCO article (aigc.bar), section "FUSCO 的核心创新": the sender reads rows
// by segment descriptor and the receiver writes each row straight into its
// final position.  The descriptor contents are not given; this library's are
// an expert-major receive buffer of T*k rows ordered by token inside each
// expert, with per-expert counts/offsets, per-rank offsets from the ceil/floor
// partition of TensorRT-LLM PR #13888, the per-(token, column) receive row
// ("slot") and, for node staging, per-node token ranks.
//
// With MOE_FLAG_LAYOUT_CLUSTER and up to kClusterMaxTokens tokens, one
// launch does it all: a thread-block cluster of up to 16 CTAs, each owning a
// contiguous token range.
//   phase 1: each CTA builds its expert (and node) histogram in shared memory;
//   cluster barrier (hardware, barrier.cluster);
//   phase 2: each CTA reads every peer's histogram through distributed shared
//            memory: the totals give expert_offsets (a block scan), the peers
//            of lower rank give this CTA's first row per expert;
//   cluster barrier (no CTA leaves while a peer may still read its histogram);
//   phase 3: the CTA ranks its tokens block by block exactly as the assign
//            kernel below does, carrying the per-expert base from block to
//            block.
// No workspace, no global atomics, no spin-waits.  Measured on B200 it is
// slower inside a CUDA-graph step than the three kernels below, whose launch
// latencies overlap through programmatic dependent launch, so it is opt-in.
//
// By default (more than one chunk of 256 tokens), count then assign with the
// scan folded in (up to 256 chunks), else three kernels; no global sort and
// no atomics on positions.  A batch of one chunk takes the cluster kernel
// with a cluster of one CTA:
//   count  : one CTA per chunk of 256 tokens builds an expert histogram (and a
//            node-touch histogram) in shared memory and writes it to the
//            workspace column of its chunk, cnt[e][chunk].
//   scan   : one CTA does an exclusive scan over cnt in expert-major,
//            chunk-minor order.  Entry (e, c) becomes expert_offsets[e] plus
//            the rows of expert e in chunks before c, which is exactly where
//            chunk c's first row of expert e goes.
//   assign : one CTA per chunk again (up to 256 chunks it also does the scan
//            for itself, reading the whole [E][C] histogram; see
//            layout_assign_scan_kernel); per-warp histograms and a scan across
//            the 8 warps give each warp its base, and inside a warp a token's
//            rank among equal experts is the popcount of the lower lanes in a
//            shared-memory lane mask for that expert.  Because a token never
//            names an expert twice, this ordering is by token index.
#include <cooperative_groups.h>

#include "layout_common.cuh"
#include "moe_kernels.h"

namespace moe {
namespace {

constexpr int kLayoutWarps = 8;
constexpr int kTokensPerCta = kLayoutWarps * 32;
constexpr int kScanThreads = 1024;
constexpr int64_t kClusterMaxTokens = 131072;
constexpr int kClusterMinTokensPerCta = 256;

struct LayoutArgs {
    const int* topk;
    int64_t T;
    int k, E, N;
    int C;          // chunks
    bool nodes;
    Partition part;
    int* cnt;       // [E][C]
    int* ncnt;      // [N][C]
    int* expert_counts;
    int* expert_offsets;
    int* rank_offsets;
    int* slot;
    int* node_counts;
    int* node_offsets;
    int* node_slot;
    int* node_src;  // [U] staging row -> token, or nullptr
    int* err;
    // the count kernel writes its histograms chunk-major ([C][E], [C][N])
    // and the assign kernel copies them whole into shared memory with bulk
    // copies (16-byte aligned workspace, small enough); otherwise they are
    // expert-major ([E][C], [N][C]) and read from global memory
    bool bulk_hist;
    bool vec_routes;  // k % 4 == 0 and topk 16-byte aligned: 16-byte route loads
    bool vec_slots;   // k % 4 == 0 and slot 16-byte aligned: 16-byte slot stores
};

// Histogram bytes the assign kernel copies into shared memory at most.
constexpr size_t kBulkHistMaxBytes = 128 * 1024;
__host__ __device__ inline size_t round16(size_t v) { return (v + 15) / 16 * 16; }

template <int KMAX>
__global__ void __launch_bounds__(kTokensPerCta) layout_count_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) int smem[];
    int* s_cnt = smem;           // [E]
    int* s_ncnt = smem + a.E;    // [N]
    unsigned char* s_node = reinterpret_cast<unsigned char*>(smem + a.E + a.N);  // [E] (nodes)
    for (int i = threadIdx.x; i < a.E + a.N; i += blockDim.x) smem[i] = 0;
    if (a.nodes) fill_node_table(s_node, a.part, a.E);
    pdl_wait();
    pdl_trigger();
    __syncthreads();

    const int64_t t = (int64_t)blockIdx.x * kTokensPerCta + threadIdx.x;
    int bits = 0;
    if (t < a.T) {
        int e[KMAX];
        bits = load_route<KMAX>(a.topk, t, a.k, a.E, e, a.vec_routes);
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
            if (e[j] >= 0) atomicAdd(&s_cnt[e[j]], 1);
        if (a.nodes) {
            uint32_t m = node_mask<KMAX>(s_node, e);
            while (m) {
                const int n = __ffs(m) - 1;
                m &= m - 1;
                atomicAdd(&s_ncnt[n], 1);
            }
        }
    }
    warp_report(a.err, bits);
    __syncthreads();
    if (a.bulk_hist) {
        // this chunk's counts as one contiguous row of the [C][E] matrix
        for (int i = threadIdx.x; i < a.E; i += blockDim.x)
            a.cnt[(int64_t)blockIdx.x * a.E + i] = s_cnt[i];
        if (a.nodes)
            for (int i = threadIdx.x; i < a.N; i += blockDim.x)
                a.ncnt[(int64_t)blockIdx.x * a.N + i] = s_ncnt[i];
    } else {
        for (int i = threadIdx.x; i < a.E; i += blockDim.x)
            a.cnt[(int64_t)i * a.C + blockIdx.x] = s_cnt[i];
        if (a.nodes)
            for (int i = threadIdx.x; i < a.N; i += blockDim.x)
                a.ncnt[(int64_t)i * a.C + blockIdx.x] = s_ncnt[i];
    }
}

// In-place exclusive scan of data[0..L) by one block: each thread owns a
// contiguous span, sums it, takes its prefix from the block scan and writes
// the running prefix back.
__device__ void block_scan_inplace(int* data, int64_t L, int* s_warp, int& total) {
    const int64_t span = (L + blockDim.x - 1) / blockDim.x;
    const int64_t beg = min(L, (int64_t)threadIdx.x * span);
    const int64_t end = min(L, beg + span);
    int sum = 0;
#pragma unroll 8
    for (int64_t i = beg; i < end; ++i) sum += data[i];
    int run = block_exclusive_scan(sum, s_warp, total);
    for (int64_t i = beg; i < end; ++i) {
        const int v = data[i];
        data[i] = run;
        run += v;
    }
}

__global__ void __launch_bounds__(kScanThreads) layout_scan_kernel(LayoutArgs a) {
    __shared__ int s_warp[32];
    pdl_trigger();
    pdl_wait();
    int total = 0;
    block_scan_inplace(a.cnt, (int64_t)a.E * a.C, s_warp, total);
    __syncthreads();
    // offset of expert e = the scanned entry of its first chunk
    auto expert_off = [&](int e) -> int {
        return e < a.E ? (a.C > 0 ? a.cnt[(int64_t)e * a.C] : 0) : total;
    };
    for (int e = threadIdx.x; e <= a.E; e += blockDim.x) {
        const int off = expert_off(e);
        a.expert_offsets[e] = off;
        if (e < a.E) a.expert_counts[e] = expert_off(e + 1) - off;
    }
    for (int r = threadIdx.x; r <= a.part.R; r += blockDim.x)
        a.rank_offsets[r] = expert_off(a.part.first_expert(r));
    if (a.nodes) {
        int ntotal = 0;
        block_scan_inplace(a.ncnt, (int64_t)a.N * a.C, s_warp, ntotal);
        __syncthreads();
        auto node_off = [&](int n) -> int {
            return n < a.N ? (a.C > 0 ? a.ncnt[(int64_t)n * a.C] : 0) : ntotal;
        };
        for (int n = threadIdx.x; n <= a.N; n += blockDim.x) {
            const int off = node_off(n);
            a.node_offsets[n] = off;
            if (n < a.N) a.node_counts[n] = node_off(n + 1) - off;
        }
    }
}

template <int KMAX>
__global__ void __launch_bounds__(kTokensPerCta) layout_assign_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) int smem[];
    int* s_wcnt = smem;                                                    // [8][E]
    unsigned* s_mask = reinterpret_cast<unsigned*>(smem + kLayoutWarps * a.E);  // [8][E]
    int* s_wn = smem + 2 * kLayoutWarps * a.E;                             // [8][N]
    const int words = 2 * kLayoutWarps * a.E + kLayoutWarps * a.N;
    for (int i = threadIdx.x; i < words; i += blockDim.x) smem[i] = 0;
    pdl_trigger();
    pdl_wait();
    __syncthreads();

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * kTokensPerCta + threadIdx.x;
    int e[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) e[j] = -1;
    uint32_t nm = 0;
    if (t < a.T) {
        load_route<KMAX>(a.topk, t, a.k, a.E, e);  // errors were reported by count
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
            if (e[j] >= 0) atomicAdd(&s_wcnt[warp * a.E + e[j]], 1);
        if (a.nodes) {
            nm = node_mask<KMAX>(a.part, e);
            uint32_t m = nm;
            while (m) {
                const int n = __ffs(m) - 1;
                m &= m - 1;
                atomicAdd(&s_wn[warp * a.N + n], 1);
            }
        }
    }
    __syncthreads();
    // per-warp bases: chunk base from the scan, then earlier warps' counts
    for (int i = threadIdx.x; i < a.E; i += blockDim.x) {
        int run = a.cnt[(int64_t)i * a.C + blockIdx.x];
#pragma unroll
        for (int w = 0; w < kLayoutWarps; ++w) {
            const int v = s_wcnt[w * a.E + i];
            s_wcnt[w * a.E + i] = run;
            run += v;
        }
    }
    if (a.nodes) {
        for (int i = threadIdx.x; i < a.N; i += blockDim.x) {
            int run = a.ncnt[(int64_t)i * a.C + blockIdx.x] - a.ncnt[(int64_t)i * a.C];
#pragma unroll
            for (int w = 0; w < kLayoutWarps; ++w) {
                const int v = s_wn[w * a.N + i];
                s_wn[w * a.N + i] = run;
                run += v;
            }
        }
    }
    __syncthreads();
    // rank among the lower lanes of this warp that chose the same expert
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
        if (e[j] >= 0) atomicOr(&s_mask[warp * a.E + e[j]], 1u << lane);
    __syncwarp();
    const unsigned lt = lanemask_lt();
    if (t < a.T) {
        int* out = a.slot + t * a.k;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j < a.k) {
                int s = -1;
                if (e[j] >= 0) {
                    const int idx = warp * a.E + e[j];
                    s = s_wcnt[idx] + __popc(s_mask[idx] & lt);
                }
                out[j] = s;
            }
        }
    }
    if (a.nodes) {
        // lane n: first staging row of node n (the scanned node histogram)
        const int noff = (a.node_src && lane < a.N) ? a.ncnt[(int64_t)lane * a.C] : 0;
        for (int n = 0; n < a.N; ++n) {
            const bool touched = (nm >> n) & 1u;
            const unsigned b = __ballot_sync(kFullMask, touched);
            const int ns = touched ? s_wn[warp * a.N + n] + __popc(b & lt) : -1;
            const int off = __shfl_sync(kFullMask, noff, n);
            if (t < a.T) {
                a.node_slot[t * a.N + n] = ns;
                if (a.node_src && touched) a.node_src[off + ns] = (int)t;
            }
        }
    }
}

// Assign with the scan folded in (up to kFusedScanMaxChunks chunks): each CTA
// reads the whole [E][C] histogram the count kernel wrote, so it finds the
// totals (and from them expert_offsets) and the rows of each expert in
// earlier chunks itself; CTA 0 also writes the offsets.  One kernel boundary
// less than count / scan / assign.  The routes are read and counted before
// waiting for the count kernel: topk_idx was written before the layout
// began, and the count kernel waits for its writer before it lets this grid
// launch.  It lets its dependent grid launch only after the histogram reads.
// Shared memory (ints): tot[E+N] base[E+N] wcnt[8][E] mask[8][E] wn[8][N],
// then (bulk_hist) the [E][C] histogram and the [N][C] node histogram, each
// padded to 16 bytes, and an mbarrier.
constexpr int kFusedScanMaxChunks = 256;

// Offset (ints) of the copied histograms in the assign kernel's shared
// memory: after the fixed part, rounded up to a multiple of 4 ints.
__host__ __device__ inline int assign_scan_hist_offset(int E, int N) {
    return (2 * (E + N) + 2 * kLayoutWarps * E + kLayoutWarps * N + 3) & ~3;
}

template <int KMAX>
__global__ void __launch_bounds__(kTokensPerCta) layout_assign_scan_kernel(LayoutArgs a) {
    __shared__ int s_warp[32];
    extern __shared__ __align__(16) int smem[];
    const int E = a.E, N = a.N, EN = a.E + a.N, C = a.C;
    int* tot = smem;
    int* base = tot + EN;
    int* s_wcnt = base + EN;
    unsigned* s_mask = reinterpret_cast<unsigned*>(s_wcnt + kLayoutWarps * E);
    int* s_wn = reinterpret_cast<int*>(s_mask + kLayoutWarps * E);
    const int words = 2 * kLayoutWarps * E + kLayoutWarps * N;
    const size_t hist_e = round16(sizeof(int) * (size_t)E * C);
    const size_t hist_n = a.nodes ? round16(sizeof(int) * (size_t)N * C) : 0;
    // the copied histograms start at the next 16-byte boundary, then the
    // mbarrier (16 bytes kept), then the table of each expert's node
    int* s_hist = smem + assign_scan_hist_offset(E, N);
    uint64_t* bar = reinterpret_cast<uint64_t*>(reinterpret_cast<char*>(s_hist) +
                                                (a.bulk_hist ? hist_e + hist_n : 0));
    unsigned char* s_node = reinterpret_cast<unsigned char*>(bar + 2);
    for (int i = threadIdx.x; i < words; i += blockDim.x) s_wcnt[i] = 0;
    if (a.nodes) fill_node_table(s_node, a.part, E);
    if (a.bulk_hist && threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_barrier_init();
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * kTokensPerCta + threadIdx.x;
    int e[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) e[j] = -1;
    uint32_t nm = 0;
    if (t < a.T) {
        load_route<KMAX>(a.topk, t, a.k, E, e, a.vec_routes);  // errors were reported by count
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
            if (e[j] >= 0) {
                atomicAdd(&s_wcnt[warp * E + e[j]], 1);
                atomicOr(&s_mask[warp * E + e[j]], 1u << lane);
            }
        if (a.nodes) {
            nm = node_mask<KMAX>(s_node, e);
            uint32_t m = nm;
            while (m) {
                const int n = __ffs(m) - 1;
                m &= m - 1;
                atomicAdd(&s_wn[warp * N + n], 1);
            }
        }
    }
    pdl_wait();
    if (a.bulk_hist && threadIdx.x == 0) {
        mbar_arrive_expect_tx(bar, (uint32_t)(hist_e + hist_n));
        bulk_load(s_hist, a.cnt, (uint32_t)hist_e, bar);
        if (hist_n) bulk_load(reinterpret_cast<char*>(s_hist) + hist_e, a.ncnt, (uint32_t)hist_n, bar);
    }

    // totals and earlier-chunk rows of each expert / node.  Bulk path: one
    // round trip brings the whole histogram into shared memory; warp w then
    // reduces rows w, w + 8, ..., four rows at a time, lane l summing
    // columns l, l + 32, ... (conflict-free) and one warp reduction per row
    // for the total and one for the chunks before this CTA's.
    // Otherwise each round of loads costs an L2 round trip, so the shape of
    // the read follows C:
    //  - C <= 32: the [E+N][C] histogram is walked column-major (neighbouring
    //    threads on different rows, so their shared-memory adds do not
    //    collide), eight loads per thread in flight -- one round for E*C up
    //    to 2048;
    //  - larger C: four rows per warp, each lane summing up to 8 columns of
    //    a row and a warp reduction per row -- two rounds for E up to 64.
    for (int i = threadIdx.x; i < EN; i += blockDim.x) {
        tot[i] = 0;
        base[i] = 0;
    }
    __syncthreads();
    if (a.bulk_hist) {
        if (!__syncthreads_and(mbar_wait(bar, 0))) {
            // the copy never completed: give up on this chunk, once the copy
            // is no longer in flight (bounded), and report it
            if (threadIdx.x == 0) {
                (void)mbar_wait(bar, 0);
                atomicOr(a.err, kErrTimeout);
            }
            __syncthreads();
            return;
        }
        // thread i: expert (or node) i's column of the [C][E] ([C][N])
        // matrix, the chunks before this CTA's, then the rest
        const int* h_n = reinterpret_cast<const int*>(reinterpret_cast<const char*>(s_hist) + hist_e);
        const int cta = (int)blockIdx.x;
        for (int i = threadIdx.x; i < EN; i += blockDim.x) {
            const int* col = i < E ? s_hist + i : h_n + (i - E);
            const int stride = i < E ? E : N;
            int pre = 0, c = 0;
#pragma unroll 4
            for (; c < cta; ++c) pre += col[c * stride];
            int sum = pre;
#pragma unroll 4
            for (; c < C; ++c) sum += col[c * stride];
            tot[i] = sum;
            base[i] = pre;
        }
    } else if (C <= 32) {
        const int64_t nall = (int64_t)EN * C;
        for (int64_t f0 = threadIdx.x; f0 < nall; f0 += 8 * (int64_t)blockDim.x) {
            int v[8], row[8], col[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int64_t f = f0 + (int64_t)q * blockDim.x;
                col[q] = (int)(f / EN);
                row[q] = (int)(f - (int64_t)col[q] * EN);
                v[q] = 0;
                if (f < nall)
                    v[q] = row[q] < E ? a.cnt[(int64_t)row[q] * C + col[q]]
                                      : a.ncnt[(int64_t)(row[q] - E) * C + col[q]];
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (v[q] != 0) {
                    atomicAdd(&tot[row[q]], v[q]);
                    if (col[q] < (int)blockIdx.x) atomicAdd(&base[row[q]], v[q]);
                }
            }
        }
    } else {
        for (int i0 = warp * 4; i0 < EN; i0 += kLayoutWarps * 4) {
            int sum[4], pre[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                sum[r] = 0;
                pre[r] = 0;
                const int i = i0 + r;
                if (i < EN) {
                    const int* row = i < E ? a.cnt + (int64_t)i * C : a.ncnt + (int64_t)(i - E) * C;
#pragma unroll
                    for (int q = 0; q < kFusedScanMaxChunks / 32; ++q) {
                        const int c = lane + 32 * q;
                        if (c < C) {
                            const int v = row[c];
                            sum[r] += v;
                            pre[r] += c < (int)blockIdx.x ? v : 0;
                        }
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    sum[r] += __shfl_xor_sync(kFullMask, sum[r], o);
                    pre[r] += __shfl_xor_sync(kFullMask, pre[r], o);
                }
                if (lane == 0 && i0 + r < EN) {
                    tot[i0 + r] = sum[r];
                    base[i0 + r] = pre[r];
                }
            }
        }
    }
    __syncthreads();
    // Let the dispatch launch only now: its first loads (x rows, started
    // before it waits for this grid) would otherwise queue ahead of the
    // histogram reads above, which are this kernel's critical path.
    pdl_trigger();
    const int total = smem_exclusive_scan(tot, E, s_warp);
    const int ntotal = a.nodes ? smem_exclusive_scan(tot + E, N, s_warp) : 0;
    if (blockIdx.x == 0) {
        for (int i = threadIdx.x; i <= E; i += blockDim.x) {
            const int off = i < E ? tot[i] : total;
            a.expert_offsets[i] = off;
            if (i < E) a.expert_counts[i] = (i + 1 < E ? tot[i + 1] : total) - off;
        }
        for (int r = threadIdx.x; r <= a.part.R; r += blockDim.x) {
            const int fe = a.part.first_expert(r);
            a.rank_offsets[r] = fe < E ? tot[fe] : total;
        }
        if (a.nodes) {
            for (int i = threadIdx.x; i <= N; i += blockDim.x) {
                const int off = i < N ? tot[E + i] : ntotal;
                a.node_offsets[i] = off;
                if (i < N) a.node_counts[i] = (i + 1 < N ? tot[E + i + 1] : ntotal) - off;
            }
        }
    }
    // per-warp first rows: chunk base, then earlier warps' counts
    for (int i = threadIdx.x; i < E; i += blockDim.x) {
        int run = tot[i] + base[i];
#pragma unroll
        for (int w = 0; w < kLayoutWarps; ++w) {
            const int v = s_wcnt[w * E + i];
            s_wcnt[w * E + i] = run;
            run += v;
        }
    }
    if (a.nodes) {
        for (int i = threadIdx.x; i < N; i += blockDim.x) {
            int run = base[E + i];
#pragma unroll
            for (int w = 0; w < kLayoutWarps; ++w) {
                const int v = s_wn[w * N + i];
                s_wn[w * N + i] = run;
                run += v;
            }
        }
    }
    __syncthreads();
    const unsigned lt = lanemask_lt();
    if (t < a.T) {
        int* out = a.slot + t * a.k;
        int sl[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            sl[j] = -1;
            if (e[j] >= 0) {
                const int idx = warp * E + e[j];
                sl[j] = s_wcnt[idx] + __popc(s_mask[idx] & lt);
            }
        }
        if (a.vec_slots) {
#pragma unroll
            for (int q = 0; q < KMAX / 4; ++q)
                if (4 * q < a.k)
                    *reinterpret_cast<int4*>(out + 4 * q) =
                        make_int4(sl[4 * q], sl[4 * q + 1], sl[4 * q + 2], sl[4 * q + 3]);
        } else {
#pragma unroll
            for (int j = 0; j < KMAX; ++j)
                if (j < a.k) out[j] = sl[j];
        }
    }
    if (a.nodes) {
        for (int n = 0; n < N; ++n) {
            const bool touched = (nm >> n) & 1u;
            const unsigned b = __ballot_sync(kFullMask, touched);
            const int ns = touched ? s_wn[warp * N + n] + __popc(b & lt) : -1;
            if (t < a.T) {
                a.node_slot[t * N + n] = ns;
                if (a.node_src && touched) a.node_src[tot[E + n] + ns] = (int)t;
            }
        }
    }
}

// Whole layout in one cluster launch (see the file comment).  Shared memory
// (ints): hist[E+N] | tot[E+N] | base[E+N] | wbase[W][ES] wmask[W][ES] wn[W][N],
// W = blockDim.x / 32, ES = E rounded to an odd stride (conflict-free columns).
constexpr int kMaxCluster = 16;

template <int KMAX>
__global__ void __launch_bounds__(1024) layout_cluster_kernel(LayoutArgs a, int64_t tokens_per_cta) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    __shared__ int s_warp[32];
    extern __shared__ __align__(16) int smem[];
    const int E = a.E, N = a.N, EN = a.E + a.N;
    const int ES = (E & 1) ? E : E + 1;
    const int W = blockDim.x >> 5;
    int* hist = smem;
    int* tot = hist + EN;
    int* base = tot + EN;
    int* wbase = base + EN;
    unsigned* wmask = reinterpret_cast<unsigned*>(wbase + W * ES);
    int* wn = reinterpret_cast<int*>(wmask + W * ES);

    const int rank = (int)cluster.block_rank();
    const int csize = (int)cluster.num_blocks();
    const int64_t t0 = min(a.T, (int64_t)rank * tokens_per_cta);
    const int64_t t1 = min(a.T, t0 + tokens_per_cta);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const unsigned lt = lanemask_lt();

    for (int i = tid; i < EN; i += blockDim.x) hist[i] = 0;
    pdl_wait();
    pdl_trigger();
    __syncthreads();

    // phase 1: histogram of this CTA's tokens (the first pass stays in
    // registers for phase 3 when k is small)
    constexpr bool kKeep = KMAX <= 8;
    int e0[KMAX];
    uint32_t nm0 = 0;
    int bits = 0;
    for (int64_t b0 = t0; b0 < t1; b0 += blockDim.x) {
        const int64_t t = b0 + tid;
        int e[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) e[j] = -1;
        if (t < t1) bits |= load_route<KMAX>(a.topk, t, a.k, E, e);
        uint32_t nm = a.nodes ? node_mask<KMAX>(a.part, e) : 0u;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j >= a.k) break;
            // one atomic per distinct expert among the warp's lanes
            const unsigned same = __match_any_sync(kFullMask, e[j]);
            if (e[j] >= 0 && (same & lt) == 0) atomicAdd(&hist[e[j]], __popc(same));
        }
        for (int n = 0; n < N; ++n) {
            const unsigned bal = __ballot_sync(kFullMask, (nm >> n) & 1u);
            if (lane == 0 && bal) atomicAdd(&hist[E + n], __popc(bal));
        }
        if (kKeep && b0 == t0) {
#pragma unroll
            for (int j = 0; j < KMAX; ++j) e0[j] = e[j];
            nm0 = nm;
        }
    }
    warp_report(a.err, bits);
    cluster.sync();

    // phase 2: totals and this CTA's bases from every peer's histogram
    for (int i = tid; i < EN; i += blockDim.x) {
        int v[kMaxCluster];
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r)
            v[r] = r < csize ? cluster.map_shared_rank(hist, r)[i] : 0;
        int all = 0, before = 0;
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r) {
            all += v[r];
            before += r < rank ? v[r] : 0;
        }
        tot[i] = all;
        base[i] = before;
    }
    cluster.sync();
    // counts into hist[] (peers no longer read it), offsets into tot[]
    for (int i = tid; i < EN; i += blockDim.x) hist[i] = tot[i];
    __syncthreads();
    const int total = smem_exclusive_scan(tot, E, s_warp);
    const int ntotal = a.nodes ? smem_exclusive_scan(tot + E, N, s_warp) : 0;
    for (int i = tid; i < E; i += blockDim.x) base[i] += tot[i];
    if (rank == 0) {
        for (int i = tid; i <= E; i += blockDim.x) {
            a.expert_offsets[i] = i < E ? tot[i] : total;
            if (i < E) a.expert_counts[i] = hist[i];
        }
        for (int r = tid; r <= a.part.R; r += blockDim.x) {
            const int fe = a.part.first_expert(r);
            a.rank_offsets[r] = fe < E ? tot[fe] : total;
        }
        if (a.nodes) {
            for (int i = tid; i <= N; i += blockDim.x) {
                a.node_offsets[i] = i < N ? tot[E + i] : ntotal;
                if (i < N) a.node_counts[i] = hist[E + i];
            }
        }
    }
    __syncthreads();

    // phase 3: stable ranks, one block of blockDim.x tokens at a time.  A
    // warp's count of expert e is the popcount of its lane mask for e; a scan
    // of those counts across warps (one warp-shuffle scan per expert) gives
    // each warp its first row.
    int* my_base = wbase + warp * ES;
    unsigned* my_mask = wmask + warp * ES;
    for (int64_t b0 = t0; b0 < t1; b0 += blockDim.x) {
        for (int i = lane; i < E; i += 32) my_mask[i] = 0u;
        __syncwarp();
        const int64_t t = b0 + tid;
        int e[KMAX];
        uint32_t nm;
        if (kKeep && b0 == t0) {
#pragma unroll
            for (int j = 0; j < KMAX; ++j) e[j] = e0[j];
            nm = nm0;
        } else {
#pragma unroll
            for (int j = 0; j < KMAX; ++j) e[j] = -1;
            if (t < t1) load_route<KMAX>(a.topk, t, a.k, E, e);
            nm = a.nodes ? node_mask<KMAX>(a.part, e) : 0u;
        }
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
            if (e[j] >= 0) atomicOr(&my_mask[e[j]], 1u << lane);
        for (int n = 0; n < N; ++n) {
            const unsigned bal = __ballot_sync(kFullMask, (nm >> n) & 1u);
            if (lane == 0) wn[warp * N + n] = __popc(bal);
        }
        __syncthreads();
        for (int i = warp; i < EN; i += W) {
            int v = 0;
            if (lane < W) v = i < E ? __popc(wmask[lane * ES + i]) : wn[lane * N + (i - E)];
            const int incl = warp_inclusive_scan(v);
            const int b = base[i];
            if (lane < W) {
                if (i < E) wbase[lane * ES + i] = b + incl - v;
                else wn[lane * N + (i - E)] = b + incl - v;
            }
            if (lane == 31) base[i] = b + incl;
        }
        __syncthreads();
        if (t < t1) {
            int* out = a.slot + t * a.k;
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (j < a.k)
                    out[j] = e[j] >= 0 ? my_base[e[j]] + __popc(my_mask[e[j]] & lt) : -1;
            }
        }
        for (int n = 0; n < N; ++n) {
            const bool touched = (nm >> n) & 1u;
            const unsigned bal = __ballot_sync(kFullMask, touched);
            const int ns = touched ? wn[warp * N + n] + __popc(bal & lt) : -1;
            if (t < t1) {
                a.node_slot[t * N + n] = ns;
                if (a.node_src && touched) a.node_src[tot[E + n] + ns] = (int)t;
            }
        }
        __syncthreads();
    }
}

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

template <int KMAX>
cudaError_t launch_layout_k(const LayoutArgs& a, cudaStream_t stream) {
    cudaError_t err;
    if (a.C > 0) {
        const size_t smem = sizeof(int) * (size_t)(a.E + a.N) + (a.nodes ? (size_t)a.E : 0);
        err = launch_pdl(layout_count_kernel<KMAX>, dim3(a.C), dim3(kTokensPerCta), smem, stream, a);
        if (err != cudaSuccess) return err;
    }
    if (a.C > 0 && a.C <= kFusedScanMaxChunks) {
        size_t smem = sizeof(int) * (size_t)assign_scan_hist_offset(a.E, a.N) + 2 * sizeof(uint64_t) +
                      (a.nodes ? (size_t)a.E : 0);
        if (a.bulk_hist)
            smem += round16(sizeof(int) * (size_t)a.E * a.C) +
                    (a.nodes ? round16(sizeof(int) * (size_t)a.N * a.C) : 0);
        if (smem > 48 * 1024) {
            err = cudaFuncSetAttribute(layout_assign_scan_kernel<KMAX>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (err != cudaSuccess) return err;
        }
        return launch_pdl(layout_assign_scan_kernel<KMAX>, dim3(a.C), dim3(kTokensPerCta), smem,
                          stream, a);
    }
    err = launch_pdl(layout_scan_kernel, dim3(1), dim3(kScanThreads), 0, stream, a);
    if (err != cudaSuccess) return err;
    if (a.C > 0) {
        const size_t smem = sizeof(int) * (size_t)(2 * kLayoutWarps * a.E + kLayoutWarps * a.N);
        if (smem > 48 * 1024) {
            err = cudaFuncSetAttribute(layout_assign_kernel<KMAX>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (err != cudaSuccess) return err;
        }
        err = launch_pdl(layout_assign_kernel<KMAX>, dim3(a.C), dim3(kTokensPerCta), smem, stream, a);
    }
    return err;
}

// Threads per CTA for the cluster kernel: no more warps than tokens need,
// and few enough that the per-warp lane masks fit in about 64 KB.
inline int cluster_threads(int E, int64_t tokens_per_cta) {
    int w = 8192 / (E > 0 ? E : 1);
    w = w > 32 ? 32 : (w < 8 ? 8 : w);
    const int64_t need = (tokens_per_cta + 31) / 32;
    if (need < w) w = need < 1 ? 1 : (int)need;
    return w * 32;
}

inline size_t cluster_smem(int E, int N, int threads) {
    const int W = threads / 32;
    const int ES = (E & 1) ? E : E + 1;
    return sizeof(int) * (size_t)(3 * (E + N) + W * (2 * ES + N));
}

// Upper bound of cluster_smem() over E <= MOE_MAX_EXPERTS (1024), N <= 32 and
// the warps cluster_threads() picks: W * 2 * ES <= 16448, W * N <= 1024,
// 3 * (E + N) <= 3168 ints, i.e. under 83 KB.
constexpr size_t kClusterSmemBound = 96 * 1024;

// Largest cluster size (16 if the device runs it, else 8) for this kernel.
template <int KMAX>
int max_cluster_size(int threads, size_t smem) {
    static int cached = 0;
    if (cached == 0) {
        cached = 8;
        auto kern = layout_cluster_kernel<KMAX>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) ==
                cudaSuccess &&
            cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                cudaSuccess) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(16);
            cfg.blockDim = dim3(threads);
            cfg.dynamicSmemBytes = smem;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 16;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int clusters = 0;
            if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) == cudaSuccess && clusters > 0)
                cached = 16;
        }
        cudaGetLastError();  // clear a refused probe
    }
    return cached;
}

template <int KMAX>
cudaError_t launch_layout_cluster(const LayoutArgs& a, cudaStream_t stream) {
    auto kern = layout_cluster_kernel<KMAX>;
    const int cmax = max_cluster_size<KMAX>(1024, kClusterSmemBound);
    int64_t csize = (a.T + kClusterMinTokensPerCta - 1) / kClusterMinTokensPerCta;
    if (csize > cmax) csize = cmax;
    if (csize < 1) csize = 1;
    const int64_t per_cta = (a.T + csize - 1) / csize;
    const int threads = cluster_threads(a.E, per_cta);
    const size_t smem = cluster_smem(a.E, a.N, threads);
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)kClusterSmemBound);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)csize);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, a, per_cta);
}

}  // namespace

size_t fused_workspace_offset(int64_t T, int E) {
    const int64_t C = (T + kTokensPerCta - 1) / kTokensPerCta;
    return round_up(sizeof(int) * (size_t)E * (size_t)C, 256);
}

size_t layout_scratch_bytes(int64_t T, int E, int N, bool nodes) {
    const int64_t C = (T + kTokensPerCta - 1) / kTokensPerCta;
    size_t b = round_up(sizeof(int) * (size_t)E * (size_t)C, 256);
    if (nodes) b += round_up(sizeof(int) * (size_t)N * (size_t)C, 256);
    return b < 256 ? 256 : b;
}

size_t layout_workspace_bytes(int64_t T, int E, int N, bool nodes) {
    if (nodes) return layout_scratch_bytes(T, E, N, nodes);
    return fused_workspace_offset(T, E) + kFusedBarrierBytes +
           round_up(sizeof(int) * (size_t)E * kFusedMaxCtas, 256);
}

cudaError_t launch_layout(const LayoutParams& p, cudaStream_t stream) {
    LayoutArgs a;
    a.topk = p.topk;
    a.T = p.T;
    a.k = p.k;
    a.E = p.E;
    a.N = p.nodes ? p.N : 0;
    a.C = (int)((p.T + kTokensPerCta - 1) / kTokensPerCta);
    a.nodes = p.nodes;
    a.part = Partition::make(p.E, p.R, p.N);
    a.cnt = static_cast<int*>(p.workspace);
    a.ncnt = reinterpret_cast<int*>(static_cast<char*>(p.workspace) +
                                    round_up(sizeof(int) * (size_t)p.E * (size_t)a.C, 256));
    a.expert_counts = p.expert_counts;
    a.expert_offsets = p.expert_offsets;
    a.rank_offsets = p.rank_offsets;
    a.slot = p.slot;
    a.node_counts = p.node_counts;
    a.node_offsets = p.node_offsets;
    a.node_slot = p.node_slot;
    a.node_src = p.nodes ? p.node_src : nullptr;
    a.err = p.err;
    {
        // the histograms start 256 bytes apart from the workspace base, so a
        // 16-byte aligned workspace makes both bulk copies aligned
        const size_t bytes = round16(sizeof(int) * (size_t)p.E * a.C) +
                             (p.nodes ? round16(sizeof(int) * (size_t)p.N * a.C) : 0);
        a.bulk_hist = reinterpret_cast<uintptr_t>(p.workspace) % 16 == 0 &&
                      bytes <= kBulkHistMaxBytes && a.C <= kFusedScanMaxChunks;
#ifdef MOE_LAYOUT_NO_BULK_HIST
        a.bulk_hist = false;  // build-time switch: the expert-major path everywhere (A/B timing)
#endif
    }
    a.vec_routes = p.k % 4 == 0 && reinterpret_cast<uintptr_t>(p.topk) % 16 == 0;
    a.vec_slots = p.k % 4 == 0 && reinterpret_cast<uintptr_t>(p.slot) % 16 == 0;
    // One chunk of tokens (T <= 256): one CTA sees every token, so the
    // single-cluster kernel (a cluster of one CTA) does the whole layout in one
    // launch, with no count kernel and no kernel boundary before the ranks.
    if ((p.cluster && p.T <= kClusterMaxTokens) || (p.T > 0 && a.C == 1))
        return p.k <= 8 ? launch_layout_cluster<8>(a, stream) : launch_layout_cluster<32>(a, stream);
    return p.k <= 8 ? launch_layout_k<8>(a, stream) : launch_layout_k<32>(a, stream);
}

}  // namespace moe

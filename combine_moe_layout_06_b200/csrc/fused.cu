// fused.cu -- layout and flat dispatch as two kernels, the assignment of
// receive rows folded into the dispatch.
//
// FUSCO article (aigc.bar), section "FUSCO 的核心创新": rows travel straight
// from where they are to their final expert positions, with the segment
// descriptors that place them worked out on the way, so no pass over the
// data precedes or follows the transfer.  Here the stable slot assignment
// happens inside the dispatch kernel, while its x-row loads are in flight.
// Both kernels split the tokens the same way: G CTAs (at most one per SM),
// CTA c owning the contiguous range [T*c/G, T*(c+1)/G).
//
//  count_scan_kernel: each CTA counts the experts of its tokens and writes
//    the histogram as column c of an [E][Gs] matrix in the workspace, then
//    takes a ticket from a counter.  The CTA that takes the last ticket (by
//    then every column is in) turns each row into its exclusive prefix over
//    the CTAs, scans the row totals into expert_offsets, writes
//    expert_counts / expert_offsets / rank_offsets and resets the counter.
//    Nothing waits for anything: the last CTA does the work the others
//    leave.
//
//  assign_dispatch_kernel: launched as soon as the count kernel has passed
//    its own wait for the previous kernel (programmatic dependent launch),
//    so x and topk_idx are complete.  Before it waits for the count kernel,
//    every warp starts cp.async.bulk loads of its first x-row chunks into
//    its shared-memory ring and the CTA copies its routes into shared
//    memory.  After the wait it reads its column of prefixes and the expert
//    offsets (2E values), ranks its tokens stably as the assign kernel of
//    layout.cu does (per-warp lane masks, a scan across warps), writes
//    slot[], and stores each landed chunk to its k receive rows with
//    cp.async.bulk shared->global copies.
//
// Results equal moe_layout() followed by moe_dispatch() bit for bit.  The
// ticket counter lives in the workspace: it must be zero before the first
// launch, and every launch leaves it zero.  Each CTA issues its own bulk loads.
#include "layout_common.cuh"
#include "moe_kernels.h"

namespace moe {
namespace {

// Ring shape (compile-time tunables): kFStagesMax stages of kFChunk bytes
// per warp.
#ifndef MOE_FUSED_STAGES
#define MOE_FUSED_STAGES 4
#endif
#ifndef MOE_FUSED_CHUNK
#define MOE_FUSED_CHUNK 4096
#endif
constexpr int kFWarps = 12;
constexpr int kFThreads = kFWarps * 32;
constexpr int kFStagesMax = MOE_FUSED_STAGES;
constexpr uint32_t kFChunk = MOE_FUSED_CHUNK;
static_assert(kFStagesMax >= 2 && kFStagesMax <= 32, "ring stages");
static_assert(kFChunk % 16 == 0, "bulk copies move multiples of 16 bytes");
constexpr int kCWarps = 16;
constexpr int kCThreads = kCWarps * 32;
constexpr int64_t kFMinTokensPerCta = 16;
static_assert(kFusedMaxCtas <= 256 && kFusedMaxCtas % 8 == 0, "eight columns per lane in the row scan");

struct FusedArgs {
    const int* topk;
    const char* x;
    char* recv;
    int64_t T;
    int k, E, G;
    int Gs;            // row stride of cnt: G rounded up to a multiple of 8
    int stages;        // ring stages per warp (<= kFStagesMax)
    int slot_cap;      // route / slot entries per CTA (>= max tokens per CTA * k)
    Partition part;
    int64_t row_bytes;
    uint32_t chunk;    // bytes per row chunk (multiple of 16)
    int64_t cpr;       // chunks per row
    int* cnt;          // [E][Gs]: histogram columns, then their exclusive prefixes (workspace)
    unsigned* ticket;  // last-CTA counter (workspace, zero between launches)
    int* expert_counts;
    int* expert_offsets;
    int* rank_offsets;
    int* slot;
    int* err;
};

__device__ __forceinline__ int64_t range_begin(const FusedArgs& a, int c) { return a.T * c / a.G; }

// 16-byte load cached in L2 only (.cg): served by L2, never by a stale L1
// line; 16-byte aligned address.
__device__ __forceinline__ int4 ld_cg_v4(const int* p) {
    int4 v;
    asm volatile("ld.global.cg.v4.s32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ void st_v4(int* p, int4 v) {
    asm volatile("st.global.v4.s32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ unsigned ticket_acq_rel(unsigned* p) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
    return old;
}

template <int KMAX>
__global__ void __launch_bounds__(kCThreads) count_scan_kernel(FusedArgs a) {
    extern __shared__ int csm[];
    __shared__ int s_warp[32];
    __shared__ int s_last;
    const int E = a.E;
    int* hist = csm;      // [E]
    int* tot = csm + E;   // [E]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < E; i += kCThreads) hist[i] = 0;
    pdl_wait();     // topk_idx may come from the previous kernel
    pdl_trigger();  // the assign/dispatch kernel may start loading x and routes
    __syncthreads();

    const int c = blockIdx.x;
    const int64_t t0 = range_begin(a, c), t1 = range_begin(a, c + 1);
    int bits = 0;
    for (int64_t b0 = t0; b0 < t1; b0 += kCThreads) {
        const int64_t t = b0 + tid;
        int e[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) e[j] = -1;
        if (t < t1) bits |= load_route<KMAX>(a.topk, t, a.k, E, e);
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
            if (e[j] >= 0) atomicAdd(&hist[e[j]], 1);
    }
    warp_report(a.err, bits);
    __syncthreads();
    for (int i = tid; i < E; i += kCThreads) a.cnt[(int64_t)i * a.Gs + c] = hist[i];
    __syncthreads();
    // The ticket is taken with acquire-release semantics at GPU scope: it
    // releases this CTA's column (ordered before it by the block barrier)
    // and, for the last CTA, acquires every other CTA's column.
    if (tid == 0) s_last = ticket_acq_rel(a.ticket) == (unsigned)a.G - 1;
    __syncthreads();
    if (!s_last) return;

    // The last CTA: each row of the matrix becomes its exclusive prefix over
    // the CTAs.  A warp takes four rows at a time; lane l holds columns
    // [8l, 8l+8) of a row (two 16-byte loads), all eight loads of the four
    // rows in flight before any is summed.
    for (int i0 = warp * 4; i0 < E; i0 += kCWarps * 4) {
        int4 v[4][2];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int col = 8 * lane + 4 * h;
                v[r][h] = (i0 + r < E && col < a.G) ? ld_cg_v4(a.cnt + (int64_t)(i0 + r) * a.Gs + col)
                                                     : make_int4(0, 0, 0, 0);
            }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            int w[8] = {v[r][0].x, v[r][0].y, v[r][0].z, v[r][0].w,
                        v[r][1].x, v[r][1].y, v[r][1].z, v[r][1].w};
            int sum = 0;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (8 * lane + u >= a.G) w[u] = 0;  // padding columns are not data
                sum += w[u];
            }
            const int incl = warp_inclusive_scan(sum);
            int run = incl - sum;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int x = w[u];
                w[u] = run;
                run += x;
            }
            const int i = i0 + r;
            if (i < E) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int col = 8 * lane + 4 * h;
                    if (col < a.G)
                        st_v4(a.cnt + (int64_t)i * a.Gs + col,
                              make_int4(w[4 * h], w[4 * h + 1], w[4 * h + 2], w[4 * h + 3]));
                }
                if (lane == 31) {
                    tot[i] = incl;
                    hist[i] = incl;  // this expert's count
                }
            }
        }
    }
    __syncthreads();
    const int total = smem_exclusive_scan(tot, E, s_warp);  // tot[e] = expert_offsets[e]
    for (int i = tid; i <= E; i += kCThreads) {
        a.expert_offsets[i] = i < E ? tot[i] : total;
        if (i < E) a.expert_counts[i] = hist[i];
    }
    for (int r = tid; r <= a.part.R; r += kCThreads) {
        const int fe = a.part.first_expert(r);
        a.rank_offsets[r] = fe < E ? tot[fe] : total;
    }
    if (tid == 0) atomicExch(a.ticket, 0u);  // every other CTA has taken its ticket
}

template <int KMAX>
__global__ void __launch_bounds__(kFThreads, 1) assign_dispatch_kernel(FusedArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = a.E;
    const int ES = (E & 1) ? E : E + 1;  // odd stride: conflict-free columns
    unsigned char* ring = smem + (size_t)warp * a.stages * a.chunk;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)kFWarps * a.stages * a.chunk) +
                     warp * kFStagesMax;
    int* base = reinterpret_cast<int*>(smem + (size_t)kFWarps * a.stages * a.chunk +
                                       sizeof(uint64_t) * kFWarps * kFStagesMax);  // [E]
    unsigned* wmask = reinterpret_cast<unsigned*>(base + E);    // [W][ES]
    int* wbase = reinterpret_cast<int*>(wmask + kFWarps * ES);  // [W][ES]
    int* s_slot = wbase + kFWarps * ES;                         // [slot_cap]
    int* s_route = s_slot + a.slot_cap;                         // [slot_cap]

    const int c = blockIdx.x;
    const int64_t t0 = range_begin(a, c), t1 = range_begin(a, c + 1);
    const int64_t dst_rows = a.T * a.k;

    if (lane == 0) {
        for (int s = 0; s < a.stages; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    __syncwarp();
    pdl_trigger();

    // this warp's items: a contiguous range of the CTA's (row, chunk) pairs
    const int64_t items = (t1 - t0) * a.cpr;
    const int64_t first = items * warp / kFWarps;
    const int64_t mine = items * (warp + 1) / kFWarps - first;
    auto geometry = [&](int64_t q, int64_t& row, int64_t& off, uint32_t& bytes) {
        const int64_t it = first + q;
        const int64_t r = it / a.cpr;
        row = t0 + r;
        off = (it - r * a.cpr) * (int64_t)a.chunk;
        const int64_t left = a.row_bytes - off;
        bytes = left < (int64_t)a.chunk ? (uint32_t)left : a.chunk;
    };
    auto issue = [&](int64_t q) {
        const int s = (int)(q % a.stages);
        int64_t row, off;
        uint32_t bytes;
        geometry(q, row, off, bytes);
        if (lane == 0) {
            mbar_arrive_expect_tx(&full[s], bytes);
            bulk_load(ring + (size_t)s * a.chunk, a.x + row * a.row_bytes + off, bytes, &full[s]);
        }
    };

    // x rows and routes were complete before the count kernel began (it
    // waited for their writer before letting this grid launch): load them
    // before waiting for the count kernel.
    const int nroute = (int)((t1 - t0) * a.k);
    for (int i = tid; i < nroute; i += kFThreads) async_copy4(s_route + i, a.topk + t0 * a.k + i);
    async_commit();
    uint32_t parity = 0, inflight = 0;
    for (int64_t q = 0; q < a.stages && q < mine; ++q) {
        issue(q);
        inflight |= 1u << q;
    }
    async_wait<0>();
    __syncthreads();
    auto route = [&](int64_t t, int (&e)[KMAX]) {
        int raw[KMAX];
        const int* r = s_route + (t - t0) * a.k;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) raw[j] = j < a.k ? r[j] : -1;
        (void)check_route<KMAX>(raw, a.k, E, e);  // the count kernel reported errors
    };

    // first row of each expert for this CTA: expert_offsets[e] plus the rows
    // of expert e in the CTAs before this one
    pdl_wait();
    for (int i = tid; i < E; i += kFThreads)
        base[i] = ld_dep(a.expert_offsets + i) + ld_dep(a.cnt + (int64_t)i * a.Gs + c);
    __syncthreads();

    // stable ranks, one block of kFThreads tokens at a time: a warp's count
    // of expert e is the popcount of its lane mask for e, and a scan of those
    // counts across warps gives each warp its first row
    const unsigned lt = lanemask_lt();
    int* my_base = wbase + warp * ES;
    unsigned* my_mask = wmask + warp * ES;
    for (int64_t b0 = t0; b0 < t1; b0 += kFThreads) {
        for (int i = lane; i < E; i += 32) my_mask[i] = 0u;
        __syncwarp();
        const int64_t t = b0 + tid;
        int e[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) e[j] = -1;
        if (t < t1) route(t, e);
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
            if (e[j] >= 0) atomicOr(&my_mask[e[j]], 1u << lane);
        __syncthreads();
        for (int i = warp; i < E; i += kFWarps) {
            const int b = base[i];
            const int v = lane < kFWarps ? __popc(wmask[lane * ES + i]) : 0;
            const int incl = warp_inclusive_scan(v);
            if (lane < kFWarps) wbase[lane * ES + i] = b + incl - v;
            __syncwarp();
            if (lane == 31) base[i] = b + incl;
        }
        __syncthreads();
        if (t < t1) {
            int* out = a.slot + t * a.k;
            int* cache = s_slot + (t - t0) * a.k;
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (j < a.k) {
                    const int sl = e[j] >= 0 ? my_base[e[j]] + __popc(my_mask[e[j]] & lt) : -1;
                    out[j] = sl;
                    cache[j] = sl;
                }
            }
        }
        __syncthreads();
    }

    // move the rows: each landed chunk goes to the token's k receive rows
    int errbits = 0;
    for (int64_t q = 0; q < mine; ++q) {
        const int s = (int)(q % a.stages);
        if (!__all_sync(kFullMask, mbar_wait(&full[s], (parity >> s) & 1u))) {
            errbits |= kErrTimeout;
            for (int u = 0; u < a.stages; ++u)  // stage s included: its load is still in flight
                if (inflight & (1u << u)) (void)mbar_wait(&full[u], (parity >> u) & 1u);
            break;
        }
        parity ^= 1u << s;
        inflight &= ~(1u << s);
        int64_t row, off;
        uint32_t bytes;
        geometry(q, row, off, bytes);
        if (lane < a.k) {
            const int sl = s_slot[(row - t0) * a.k + lane];
            if (sl >= 0 && sl < dst_rows)
                bulk_store(a.recv + (int64_t)sl * a.row_bytes + off, ring + (size_t)s * a.chunk, bytes);
            else if (sl != -1)
                errbits |= kErrBadLayout;
        }
        bulk_commit();
        // the stage of item q-1 is free once its stores have read it
        bulk_wait_read<1>();
        __syncwarp();
        if (q >= 1 && q - 1 + a.stages < mine) {
            issue(q - 1 + a.stages);
            inflight |= 1u << ((q - 1) % a.stages);
        }
    }
    bulk_wait_all();
    warp_report(a.err, errbits);
}

struct FusedPlan {
    int G = 0, stages = 0, slot_cap = 0;
    uint32_t chunk = 0;
    size_t smem = 0;
};

size_t fused_smem(int E, int stages, uint32_t chunk, int slot_cap) {
    const int ES = (E & 1) ? E : E + 1;
    return (size_t)kFWarps * stages * chunk + sizeof(uint64_t) * kFWarps * kFStagesMax +
           sizeof(int) * ((size_t)E + (size_t)2 * kFWarps * ES + (size_t)2 * slot_cap);
}

// Launch shape for the problem, or G == 0 when these kernels do not apply
// (too many experts, or shared memory too small for the route cache).
FusedPlan fused_plan(int64_t T, int k, int E, size_t row_bytes) {
    FusedPlan p;
    if (T <= 0 || k < 1 || k > kFusedMaxTopk || E > kFusedMaxExperts) return p;
    int dev = 0, optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return p;
    int64_t G = (T + kFMinTokensPerCta - 1) / kFMinTokensPerCta;
    const int64_t sms = device_sm_count();
    if (G > sms) G = sms;
    if (G > kFusedMaxCtas) G = kFusedMaxCtas;
    if (G < 1) G = 1;
    const int64_t per_cta = (T + G - 1) / G;
    if (per_cta * k > (int64_t)1 << 20) return p;
    const int slot_cap = (int)(per_cta * k);
    const uint32_t chunk = (size_t)kFChunk < row_bytes ? kFChunk : (uint32_t)row_bytes;
    for (int stages = kFStagesMax; stages >= 2; --stages) {
        const size_t smem = fused_smem(E, stages, chunk, slot_cap);
        if (smem <= (size_t)optin) {
            p.G = (int)G;
            p.stages = stages;
            p.slot_cap = slot_cap;
            p.chunk = chunk;
            p.smem = smem;
            return p;
        }
    }
    return p;
}

template <int KMAX>
cudaError_t launch_fused_k(const FusedArgs& a, size_t smem, cudaStream_t stream) {
    cudaError_t e = launch_pdl(count_scan_kernel<KMAX>, dim3((unsigned)a.G), dim3(kCThreads),
                               sizeof(int) * 2 * (size_t)a.E, stream, a);
    if (e != cudaSuccess) return e;
    auto kern = assign_dispatch_kernel<KMAX>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3((unsigned)a.G), dim3(kFThreads), smem, stream, a);
}

}  // namespace

bool layout_dispatch_fused_eligible(int64_t T, int k, int E, size_t row_bytes) {
    return fused_plan(T, k, E, row_bytes).G > 0;
}

cudaError_t launch_layout_dispatch_fused(const LayoutParams& lp, const void* x, void* recv,
                                         size_t row_bytes, cudaStream_t stream) {
    const FusedPlan plan = fused_plan(lp.T, lp.k, lp.E, row_bytes);
    if (plan.G == 0) return cudaErrorInvalidValue;
    FusedArgs a;
    a.topk = lp.topk;
    a.x = static_cast<const char*>(x);
    a.recv = static_cast<char*>(recv);
    a.T = lp.T;
    a.k = lp.k;
    a.E = lp.E;
    a.G = plan.G;
    a.Gs = (plan.G + 7) & ~7;
    a.stages = plan.stages;
    a.slot_cap = plan.slot_cap;
    a.part = Partition::make(lp.E, lp.R, 1);
    a.row_bytes = (int64_t)row_bytes;
    a.chunk = plan.chunk;
    a.cpr = (a.row_bytes + a.chunk - 1) / a.chunk;
    char* fused = static_cast<char*>(lp.workspace) + fused_workspace_offset(lp.T, lp.E);
    a.ticket = reinterpret_cast<unsigned*>(fused);
    a.cnt = reinterpret_cast<int*>(fused + kFusedBarrierBytes);
    a.expert_counts = lp.expert_counts;
    a.expert_offsets = lp.expert_offsets;
    a.rank_offsets = lp.rank_offsets;
    a.slot = lp.slot;
    a.err = lp.err;
    return lp.k <= 8 ? launch_fused_k<8>(a, plan.smem, stream)
                     : launch_fused_k<kFusedMaxTopk>(a, plan.smem, stream);
}

}  // namespace moe

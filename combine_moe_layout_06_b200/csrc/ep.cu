// ep.cu -- layout for expert parallelism over sharded sources.
//
// With one rank per GPU, rank g routes only its own tokens, and every rank's
// receive buffer holds its experts' rows ("[None][feat] support non-divisible
// EP in MoE alltoall and slurm benchmark", TensorRT-LLM PR #13888: the
// NVLinkOneSided dispatch writes straight into peer receive buffers; FUSCO
// article, section "FUSCO 的核心创新": each row goes straight to its final
// position).  A rank first runs the ordinary layout over its own tokens,
// which gives its per-expert counts; the counts of all ranks are exchanged
// (counts_all[G][E], an all-gather the caller runs); this kernel then turns
// each local row into a row of the concatenated receive buffers, ordered
// expert-major, then by source rank, then by the source's token order:
//
//   slot[t][j] = local_slot[t][j] - local_offsets[e] + expert_offsets[e]
//                + sum over sources h < g of counts_all[h][e],   e = topk[t][j]
//
// with expert_offsets the exclusive prefix of the expert totals over all
// sources.  Rank r's receive buffer holds rows [rank_offsets[r],
// rank_offsets[r+1]) of the concatenation.  When the shards are the source
// ranks' contiguous token ranges in rank order, these are exactly the
// single-source slots.
#include "moe_kernels.h"

namespace moe {
namespace {

constexpr int kEpThreads = 256;

struct EpArgs {
    EpParams p;
    Partition part;
};

// Exclusive scan of data[0..L) in shared memory by one block (each thread
// owns a contiguous span); returns the total.
__device__ int ep_block_scan(int* data, int L, int* s_warp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const int span = (L + blockDim.x - 1) / blockDim.x;
    const int beg = min(L, (int)threadIdx.x * span), end = min(L, beg + span);
    int sum = 0;
    for (int i = beg; i < end; ++i) sum += data[i];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFullMask, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nwarps ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFullMask, w, o);
            if (lane >= o) w += y;
        }
        s_warp[lane] = w;
    }
    __syncthreads();
    int run = (warp > 0 ? s_warp[warp - 1] : 0) + incl - sum;
    const int total = s_warp[nwarps - 1];
    for (int i = beg; i < end; ++i) {
        const int v = data[i];
        data[i] = run;
        run += v;
    }
    __syncthreads();
    return total;
}

// One CTA per chunk of kEpThreads tokens; every CTA derives the per-expert
// shift from counts_all itself (G*E ints), CTA 0 also writes the offsets.
__global__ void __launch_bounds__(kEpThreads) ep_layout_kernel(EpArgs a) {
    __shared__ int s_warp[32];
    extern __shared__ int smem[];
    const EpParams& p = a.p;
    int* off = smem;          // [E]: totals, then expert offsets
    int* shift = smem + p.E;  // [E]
    pdl_wait();
    pdl_trigger();
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        int total = 0, before = 0;
        for (int h = 0; h < p.G; ++h) {
            const int c = ld_dep(p.counts_all + (int64_t)h * p.E + e);
            total += c;
            before += h < p.g ? c : 0;
        }
        off[e] = total;
        shift[e] = before - ld_dep(p.local_expert_offsets + e);
    }
    __syncthreads();
    const int all = ep_block_scan(off, p.E, s_warp);
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) shift[e] += off[e];
    if (blockIdx.x == 0) {
        for (int e = threadIdx.x; e <= p.E; e += blockDim.x) p.expert_offsets[e] = e < p.E ? off[e] : all;
        for (int r = threadIdx.x; r <= p.R; r += blockDim.x) {
            const int fe = a.part.first_expert(r);
            p.rank_offsets[r] = fe < p.E ? off[fe] : all;
        }
    }
    __syncthreads();
    const int64_t t = (int64_t)blockIdx.x * kEpThreads + threadIdx.x;
    int bad = 0;
    if (t < p.T) {
        for (int j = 0; j < p.k; ++j) {
            const int s = ld_dep(p.local_slot + t * p.k + j);
            const int e = ld_dep(p.topk + t * p.k + j);
            int out = -1;
            if (s >= 0) {
                if (e >= 0 && e < p.E) out = s + shift[e];
                else bad = kErrBadLayout;
            }
            p.slot[t * p.k + j] = out;
        }
    }
    warp_report(p.err, bad);
}

}  // namespace

cudaError_t launch_ep_layout(const EpParams& p, cudaStream_t stream) {
    EpArgs a;
    a.p = p;
    a.part = Partition::make(p.E, p.R, 1);
    const int64_t blocks = p.T > 0 ? (p.T + kEpThreads - 1) / kEpThreads : 1;
    const size_t smem = sizeof(int) * 2 * (size_t)p.E;
    return launch_pdl(ep_layout_kernel, dim3((unsigned)blocks), dim3(kEpThreads), smem, stream, a);
}

}  // namespace moe

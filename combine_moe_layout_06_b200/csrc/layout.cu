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
// Three kernels, no global sort and no atomics on positions:
//   count  : one CTA per chunk of 256 tokens builds an expert histogram (and a
//            node-touch histogram) in shared memory and writes it to the
//            workspace column of its chunk, cnt[e][chunk].
//   scan   : one CTA does an exclusive scan over cnt in expert-major,
//            chunk-minor order.  Entry (e, c) becomes expert_offsets[e] plus
//            the rows of expert e in chunks before c, which is exactly where
//            chunk c's first row of expert e goes.
//   assign : one CTA per chunk again; per-warp histograms and a scan across
//            the 8 warps give each warp its base, and inside a warp a token's
//            rank among equal experts is the popcount of the lower lanes in a
//            shared-memory lane mask for that expert.  Because a token never
//            names an expert twice, this ordering is by token index.
#include "moe_kernels.h"

namespace moe {
namespace {

constexpr int kLayoutWarps = 8;
constexpr int kTokensPerCta = kLayoutWarps * 32;
constexpr int kScanThreads = 1024;

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
    int* err;
};

// Load token t's k expert ids.  Invalid entries become -1 and set error
// bits: an id outside [0, E), or a repeat of an id earlier in the row (the
// later copy is dropped).  Count and assign use the same rule, so the
// histogram and the ranks always agree even on bad input.
template <int KMAX>
__device__ __forceinline__ int load_route(const int* __restrict__ topk, int64_t t, int k, int E,
                                          int (&e)[KMAX]) {
    int bits = 0;
    const int* row = topk + t * k;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        int v = -1;
        if (j < k) {
            v = __ldg(row + j);
            if (v < 0 || v >= E) {
                bits |= kErrExpertOob;
                v = -1;
            }
        }
        e[j] = v;
    }
#pragma unroll
    for (int j = 1; j < KMAX; ++j) {
#pragma unroll
        for (int i = 0; i < j; ++i) {
            if (e[j] >= 0 && e[i] == e[j]) {
                bits |= kErrDupExpert;
                e[j] = -1;
            }
        }
    }
    return bits;
}

template <int KMAX>
__device__ __forceinline__ uint32_t node_mask(const Partition& part, const int (&e)[KMAX]) {
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
        if (e[j] >= 0) m |= 1u << part.node_of(e[j]);
    return m;
}

template <int KMAX>
__global__ void __launch_bounds__(kTokensPerCta) layout_count_kernel(LayoutArgs a) {
    extern __shared__ int smem[];
    int* s_cnt = smem;           // [E]
    int* s_ncnt = smem + a.E;    // [N]
    for (int i = threadIdx.x; i < a.E + a.N; i += blockDim.x) smem[i] = 0;
    pdl_wait();
    pdl_trigger();
    __syncthreads();

    const int64_t t = (int64_t)blockIdx.x * kTokensPerCta + threadIdx.x;
    int bits = 0;
    if (t < a.T) {
        int e[KMAX];
        bits = load_route<KMAX>(a.topk, t, a.k, a.E, e);
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
            if (e[j] >= 0) atomicAdd(&s_cnt[e[j]], 1);
        if (a.nodes) {
            uint32_t m = node_mask<KMAX>(a.part, e);
            while (m) {
                const int n = __ffs(m) - 1;
                m &= m - 1;
                atomicAdd(&s_ncnt[n], 1);
            }
        }
    }
    warp_report(a.err, bits);
    __syncthreads();
    for (int i = threadIdx.x; i < a.E; i += blockDim.x)
        a.cnt[(int64_t)i * a.C + blockIdx.x] = s_cnt[i];
    if (a.nodes)
        for (int i = threadIdx.x; i < a.N; i += blockDim.x)
            a.ncnt[(int64_t)i * a.C + blockIdx.x] = s_ncnt[i];
}

// Exclusive scan of one value per thread over the whole block; also returns
// the block total.  s_warp holds 32 ints.
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int& total) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFullMask, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
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
    const int before = warp > 0 ? s_warp[warp - 1] : 0;
    total = s_warp[nwarps - 1];
    __syncthreads();
    return before + x - v;
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
    pdl_wait();
    pdl_trigger();
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
    extern __shared__ int smem[];
    int* s_wcnt = smem;                                                    // [8][E]
    unsigned* s_mask = reinterpret_cast<unsigned*>(smem + kLayoutWarps * a.E);  // [8][E]
    int* s_wn = smem + 2 * kLayoutWarps * a.E;                             // [8][N]
    const int words = 2 * kLayoutWarps * a.E + kLayoutWarps * a.N;
    for (int i = threadIdx.x; i < words; i += blockDim.x) smem[i] = 0;
    pdl_wait();
    pdl_trigger();
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
        for (int n = 0; n < a.N; ++n) {
            const bool touched = (nm >> n) & 1u;
            const unsigned b = __ballot_sync(kFullMask, touched);
            if (t < a.T)
                a.node_slot[t * a.N + n] = touched ? s_wn[warp * a.N + n] + __popc(b & lt) : -1;
        }
    }
}

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

template <int KMAX>
cudaError_t launch_layout_k(const LayoutArgs& a, cudaStream_t stream) {
    cudaError_t err;
    if (a.C > 0) {
        const size_t smem = sizeof(int) * (size_t)(a.E + a.N);
        err = launch_pdl(layout_count_kernel<KMAX>, dim3(a.C), dim3(kTokensPerCta), smem, stream, a);
        if (err != cudaSuccess) return err;
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

}  // namespace

size_t layout_workspace_bytes(int64_t T, int E, int N, bool nodes) {
    const int64_t C = (T + kTokensPerCta - 1) / kTokensPerCta;
    size_t b = round_up(sizeof(int) * (size_t)E * (size_t)C, 256);
    if (nodes) b += round_up(sizeof(int) * (size_t)N * (size_t)C, 256);
    return b < 256 ? 256 : b;
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
    a.err = p.err;
    return p.k <= 8 ? launch_layout_k<8>(a, stream) : launch_layout_k<32>(a, stream);
}

}  // namespace moe

// combine.cu -- fused combine.
//
// INC-MoE abstract: combine returns the expert outputs of each token to the
// token's owner, where they are reduced by gate weight.  Here the k expert
// rows of token t are gathered straight from the expert-major buffer (the
// scatter-recv layout of the FUSCO article, section "FUSCO 的核心创新") and
// summed in fp32 registers before one bf16 store; no unpack pass runs.
//
// Arithmetic, fixed so that results are reproducible bit for bit: acc starts
// at +0.0f and, for j = 0 .. k-1 in top-k column order, acc = fma(w[t][j],
// float(eo[slot[t][j]][h]), acc) with a single rounding per step; the store
// rounds to nearest even.
//
// Work items are (token, row chunk) pairs, a chunk being 32*VPL vectors of
// the row, over a grid from persistent_grid() (resident, or whole resident
// waves for large problems); each warp takes a contiguous token-major range
// of items, so a token's k slots and weights
// (held one per lane) are loaded once, and the next token's are fetched
// while the current chunk's rows are in flight.  The chunk of up to KB
// expert rows is loaded before any FMA, so KB*VPL streaming loads per lane
// are in flight at once.
//
// Large grids (many resident waves of items) take the paired form: lane l
// owns vectors 2l and 2l+1 of the chunk and moves both with one 32-byte load
// or store (sm_100's 256-bit global accesses), which halves the load
// instructions per byte in flight.  The arithmetic is the same; only which
// lane holds which element changes.
#include "moe_kernels.h"

namespace moe {
namespace {

constexpr int kWarpsPerCta = 8;
constexpr int kThreads = kWarpsPerCta * 32;

// 16-byte vectors per lane in one row chunk (1 KB chunks) and expert rows
// loaded per batch; compile-time tunables.  Batches of 4 rows (80
// registers, 3 CTAs per SM) beat batches of 8 (127 registers, 2 CTAs per
// SM) on B200: DeepSeek-V3-shaped step 722.7 against 725.5 us, qwen3 204.8
// against 209.2 us, the others unchanged.
#ifndef MOE_COMBINE_VPL
#define MOE_COMBINE_VPL 2
#endif
#ifndef MOE_COMBINE_KB
#define MOE_COMBINE_KB 4
#endif
// items per warp in each wave of a large combine (see persistent_grid)
#ifndef MOE_COMBINE_IPW
#define MOE_COMBINE_IPW 4
#endif
// Resident waves from which the paired (32-byte) form is used; 0 = never.
// Measured on B200: it shortens the 16-wave combines (DeepSeek-V3-shaped
// 325 -> 315 us alone, long-context 211 -> 204 us) and lengthens the 1-wave
// OLMoE-shaped one (24.1 -> 26.0 us); qwen3's 4-wave step was no faster.
#ifndef MOE_COMBINE_PAIR_WAVES
#define MOE_COMBINE_PAIR_WAVES 8
#endif

struct CombArgs {
    const void* eo;
    const float* w;
    const int* slot;   // nullptr: row of (t, j) is t*k + j
    void* y;
    int64_t T;
    int k;
    int64_t rv;        // vectors per row
    int64_t row_bytes;
    int64_t eo_rows;
    int* err;
    // expert parallelism over sharded sources: the expert rows live in the
    // buffers of ep_ranks ranks, rank r holding rows [rank_offsets[r],
    // rank_offsets[r+1]) of the concatenation, at most ep_capacity each
    const void* ep_bufs[kMaxEpRanks];
    const int* rank_offsets;
    int ep_ranks;
    int64_t ep_capacity;
    int late_trigger;  // let the dependent grid launch at the end (pdl_trigger_at_end)
};

// Lane r < ep_ranks: rank r's rows [lo, hi) and its buffer (EP only).
struct EpLane {
    int lo, hi;
    unsigned long long buf;
};

// Lane j < k: expert row and gate weight of (t, j); row -1 when invalid.
// EP: also the address of the row, in the buffer of the rank holding it.
template <bool EP>
__device__ __forceinline__ void load_route(const CombArgs& a, int64_t t, int lane, const EpLane& el,
                                           int& s, float& w, unsigned long long& rowp, int& bad) {
    s = -1;
    w = 0.f;
    if (lane < a.k) {
        s = a.slot ? ld_dep(a.slot + t * a.k + lane) : (int)(t * a.k + lane);
        w = ld_dep(a.w + t * a.k + lane);
    }
    if constexpr (EP) {
        int r = 0;
        for (int q = 1; q < a.ep_ranks; ++q) r += s >= __shfl_sync(kFullMask, el.lo, q) ? 1 : 0;
        const int lo = __shfl_sync(kFullMask, el.lo, r);
        const int hi = __shfl_sync(kFullMask, el.hi, r);
        const unsigned long long buf = __shfl_sync(kFullMask, el.buf, r);
        const int64_t local = (int64_t)s - lo;
        const bool ok = s >= 0 && s < hi && local < a.ep_capacity && buf != 0ull;
        bad |= (!ok && s != -1) ? kErrBadLayout : 0;
        s = ok ? s : -1;
        rowp = ok ? buf + (unsigned long long)local * (unsigned long long)a.row_bytes : 0ull;
    } else {
        const bool ok = s >= 0 && s < a.eo_rows;
        bad |= (!ok && s != -1) ? kErrBadLayout : 0;
        s = ok ? s : -1;
        rowp = 0ull;
    }
}

// 32 contiguous bytes (two 16-byte vectors) in one access; p 32-byte aligned.
__device__ __forceinline__ void ld_stream_pair(const uint4* p, uint4& u, uint4& v) {
    asm volatile("ld.global.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w), "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
}
__device__ __forceinline__ void st_pair(uint4* p, const uint4& u, const uint4& v) {
    asm volatile("st.global.v8.u32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(u.x), "r"(u.y),
                 "r"(u.z), "r"(u.w), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// PAIR (V = uint4, VPL = 2, rv even, expert rows and y 32-byte aligned):
// lane l holds vectors 2l, 2l+1 of the chunk instead of l, l+32.
template <typename V, int VPL, int KB, bool EP = false, bool PAIR = false>
__global__ void __launch_bounds__(kThreads) combine_kernel(CombArgs a) {
    static_assert(!PAIR || (sizeof(V) == 16 && VPL == 2 && !EP), "paired form: 16-byte vectors, 2 per lane");
    constexpr int EPV = VecInfo<V>::kElems;
    constexpr int CHUNK = 32 * VPL;
    if (!a.late_trigger) pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    EpLane el = {0, 0, 0ull};
    if (EP && lane < a.ep_ranks) {
        el.lo = ld_dep(a.rank_offsets + lane);
        el.hi = ld_dep(a.rank_offsets + lane + 1);
        el.buf = reinterpret_cast<unsigned long long>(a.ep_bufs[lane]);
    }
    const int64_t cpr = (a.rv + CHUNK - 1) / CHUNK;
    const int64_t items = a.T * cpr;
    const int64_t nw = (int64_t)gridDim.x * kWarpsPerCta;
    const int64_t gw = (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    const int64_t ib = items * gw / nw, ie = items * (gw + 1) / nw;
    const V* eo = static_cast<const V*>(a.eo);
    V* y = static_cast<V*>(a.y);
    int errbits = 0;
    if (ib < ie) {
        int64_t t = ib / cpr;
        int64_t c = ib - t * cpr;
        int s, s_next = -1;
        float wl, w_next = 0.f;
        unsigned long long rp, rp_next = 0ull;
        load_route<EP>(a, t, lane, el, s, wl, rp, errbits);
        for (int64_t item = ib; item < ie; ++item) {
            const bool last_chunk = c + 1 == cpr;
            if (last_chunk && item + 1 < ie) load_route<EP>(a, t + 1, lane, el, s_next, w_next, rp_next, errbits);
            const int64_t base = c * CHUNK;
            float acc[VPL][EPV];
#pragma unroll
            for (int i = 0; i < VPL; ++i)
#pragma unroll
                for (int e = 0; e < EPV; ++e) acc[i][e] = 0.f;
            for (int j0 = 0; j0 < a.k; j0 += KB) {
                V v[KB][VPL];
                float wq[KB];
                bool ok[KB];
#pragma unroll
                for (int q = 0; q < KB; ++q) {
                    const int j = j0 + q;
                    const int sj = __shfl_sync(kFullMask, s, j & 31);
                    wq[q] = __shfl_sync(kFullMask, wl, j & 31);
                    ok[q] = j < a.k && sj >= 0;
                    const unsigned long long rj = EP ? __shfl_sync(kFullMask, rp, j & 31) : 0ull;
                    if (ok[q]) {
                        const V* row = EP ? reinterpret_cast<const V*>(rj) + base
                                          : eo + (int64_t)sj * a.rv + base;
                        if constexpr (PAIR) {
                            if (base + 2 * lane < a.rv) ld_stream_pair(row + 2 * lane, v[q][0], v[q][1]);
                        } else {
#pragma unroll
                            for (int i = 0; i < VPL; ++i)
                                if (base + i * 32 + lane < a.rv) v[q][i] = ld_stream(row + i * 32 + lane);
                        }
                    }
                }
#pragma unroll
                for (int q = 0; q < KB; ++q) {
                    if (!ok[q]) continue;
#pragma unroll
                    for (int i = 0; i < VPL; ++i) {
                        if (PAIR ? base + 2 * lane < a.rv : base + i * 32 + lane < a.rv) {
                            float f[EPV];
                            unpack_bf16<V>(v[q][i], f);
#pragma unroll
                            for (int e = 0; e < EPV; ++e) acc[i][e] = __fmaf_rn(wq[q], f[e], acc[i][e]);
                        }
                    }
                }
            }
            V* yrow = y + t * a.rv + base;
            if constexpr (PAIR) {
                if (base + 2 * lane < a.rv) st_pair(yrow + 2 * lane, pack_bf16<V>(acc[0]), pack_bf16<V>(acc[1]));
            } else {
#pragma unroll
                for (int i = 0; i < VPL; ++i)
                    if (base + i * 32 + lane < a.rv) yrow[i * 32 + lane] = pack_bf16<V>(acc[i]);
            }
            if (last_chunk) {
                s = s_next;
                wl = w_next;
                rp = rp_next;
                ++t;
                c = 0;
            } else {
                ++c;
            }
        }
    }
    if (a.late_trigger) pdl_trigger();
    warp_report(a.err, errbits);
}

template <auto Kern>
cudaError_t launch_combine_grid(CombArgs a, int64_t items, cudaStream_t stream) {
    const int grid = persistent_grid<Kern>(items, kThreads, 0, MOE_COMBINE_IPW);
    a.late_trigger = pdl_trigger_at_end(grid, resident_blocks<Kern>(kThreads)) ? 1 : 0;
    return launch_pdl(Kern, dim3(grid), dim3(kThreads), 0, stream, a);
}

template <typename V, int VPL, int KB, bool EP>
cudaError_t launch_combine_v(CombArgs a, cudaStream_t stream) {
    constexpr auto kern = combine_kernel<V, VPL, KB, EP>;
    const int64_t cpr = (a.rv + 32 * VPL - 1) / (32 * VPL);
    const int64_t items = a.T * cpr;
    if constexpr (!EP && VPL == 2 && sizeof(V) == 16) {
        constexpr auto paired = combine_kernel<V, VPL, KB, EP, true>;
        const uintptr_t align = reinterpret_cast<uintptr_t>(a.eo) | reinterpret_cast<uintptr_t>(a.y);
        const int64_t wave_items = (int64_t)resident_blocks<paired>(kThreads) * kWarpsPerCta * MOE_COMBINE_IPW;
        if (MOE_COMBINE_PAIR_WAVES > 0 && a.rv % 2 == 0 && align % 32 == 0 &&
            items >= (int64_t)MOE_COMBINE_PAIR_WAVES * wave_items)
            return launch_combine_grid<paired>(a, items, stream);
    }
    return launch_combine_grid<kern>(a, items, stream);
}

template <typename V, int VPL, bool EP = false>
cudaError_t launch_combine_k(CombArgs a, cudaStream_t stream) {
    constexpr int kSmall = MOE_COMBINE_KB < 4 ? MOE_COMBINE_KB : 4;
    if (a.k <= 4) return launch_combine_v<V, VPL, kSmall, EP>(a, stream);
    return launch_combine_v<V, VPL, MOE_COMBINE_KB, EP>(a, stream);
}

CombArgs comb_args(const CombineParams& p, const void* expert_out, void* y) {
    CombArgs a = {};
    a.eo = expert_out;
    a.w = p.w;
    a.slot = p.slot;
    a.y = y;
    a.T = p.T;
    a.k = p.k;
    a.row_bytes = (int64_t)p.row_bytes;
    a.eo_rows = p.T * p.k;
    a.err = p.err;
    a.rv = 0;
    return a;
}

// ---- reduce-scatter formulation (comparison path) -------------------------
// INC-MoE abstract: combine as a ReduceScatter; TensorRT-LLM PR #13888: the
// AllGather + ReduceScatter fallback.  On one GPU: every virtual rank r
// first sums, for every token, its own experts' rows (fp32, FMA in column
// order) into partial[r][t]; the partials are then added in rank order and
// rounded once.

template <int EPV>
__device__ __forceinline__ void store_f32(float* p, const float (&f)[EPV]) {
    if constexpr (EPV == 8) {
        reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
        reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
    } else if constexpr (EPV == 2) {
        *reinterpret_cast<float2*>(p) = make_float2(f[0], f[1]);
    } else {
        p[0] = f[0];
    }
}

template <int EPV>
__device__ __forceinline__ void load_f32(const float* p, float (&f)[EPV]) {
    if constexpr (EPV == 8) {
        const float4 a = reinterpret_cast<const float4*>(p)[0];
        const float4 b = reinterpret_cast<const float4*>(p)[1];
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    } else if constexpr (EPV == 2) {
        const float2 a = *reinterpret_cast<const float2*>(p);
        f[0] = a.x; f[1] = a.y;
    } else {
        f[0] = p[0];
    }
}

struct RankArgs {
    CombArgs c;
    int R;
    const int* rank_offsets;
    float* partial;       // [R*T][H] fp32
};

// Items (r, t, chunk), rank-major; a warp per item.
template <typename V>
__global__ void __launch_bounds__(kThreads) rank_partial_kernel(RankArgs ra) {
    constexpr int EPV = VecInfo<V>::kElems;
    const CombArgs& a = ra.c;
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t cpr = (a.rv + 31) / 32;
    const int64_t items = (int64_t)ra.R * a.T * cpr;
    const int64_t nw = (int64_t)gridDim.x * kWarpsPerCta;
    const int64_t H = a.rv * EPV;
    int errbits = 0;
    for (int64_t item = (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5); item < items; item += nw) {
        const int64_t row = item / cpr;                 // r*T + t
        const int64_t base = (item - row * cpr) * 32;
        const int r = (int)(row / a.T);
        const int64_t t = row - (int64_t)r * a.T;
        const int lo = ld_dep(ra.rank_offsets + r), hi = ld_dep(ra.rank_offsets + r + 1);
        int s = -1;
        float wl = 0.f;
        unsigned long long unused;
        load_route<false>(a, t, lane, EpLane{0, 0, 0ull}, s, wl, unused, errbits);
        float acc[EPV];
#pragma unroll
        for (int e = 0; e < EPV; ++e) acc[e] = 0.f;
        const int64_t idx = base + lane;
        for (int j = 0; j < a.k; ++j) {
            const int sj = __shfl_sync(kFullMask, s, j);
            const float wj = __shfl_sync(kFullMask, wl, j);
            if (sj < lo || sj >= hi || idx >= a.rv) continue;
            float f[EPV];
            unpack_bf16<V>(ld_stream(static_cast<const V*>(a.eo) + (int64_t)sj * a.rv + idx), f);
#pragma unroll
            for (int e = 0; e < EPV; ++e) acc[e] = __fmaf_rn(wj, f[e], acc[e]);
        }
        if (idx < a.rv) store_f32<EPV>(ra.partial + row * H + idx * EPV, acc);
    }
    warp_report(a.err, errbits);
}

template <typename V>
__global__ void __launch_bounds__(kThreads) rank_reduce_kernel(RankArgs ra) {
    constexpr int EPV = VecInfo<V>::kElems;
    const CombArgs& a = ra.c;
    pdl_trigger();
    pdl_wait();
    const int64_t n = a.T * a.rv;                      // output vectors
    const int64_t H = a.rv * EPV;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const int64_t t = i / a.rv, v = i - t * a.rv;
        float acc[EPV];
#pragma unroll
        for (int e = 0; e < EPV; ++e) acc[e] = 0.f;
        for (int r = 0; r < ra.R; ++r) {
            float f[EPV];
            load_f32<EPV>(ra.partial + ((int64_t)r * a.T + t) * H + v * EPV, f);
#pragma unroll
            for (int e = 0; e < EPV; ++e) acc[e] = acc[e] + f[e];
        }
        static_cast<V*>(a.y)[i] = pack_bf16<V>(acc);
    }
}

inline int vec_bytes(size_t row_bytes, const void* a, const void* b) {
    const uintptr_t bits = row_bytes | reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b);
    if (bits % 16 == 0) return 16;
    if (bits % 4 == 0) return 4;
    return 2;
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, const void* expert_out, void* y,
                           cudaStream_t stream) {
    if (p.T <= 0) return cudaSuccess;
    // register engine unless the bulk engine is asked for
    if (p.engine == CopyEngine::kBulk && bulk_eligible(p.row_bytes, {expert_out, y}))
        return launch_combine_bulk(p, expert_out, y, stream);
    CombArgs a = comb_args(p, expert_out, y);
    switch (vec_bytes(p.row_bytes, expert_out, y)) {
        case 16:
            a.rv = (int64_t)(p.row_bytes / 16);
            return launch_combine_k<uint4, MOE_COMBINE_VPL>(a, stream);
        case 4:
            a.rv = (int64_t)(p.row_bytes / 4);
            return launch_combine_k<uint32_t, 4>(a, stream);
        default:
            a.rv = (int64_t)(p.row_bytes / 2);
            return launch_combine_k<uint16_t, 4>(a, stream);
    }
}

cudaError_t launch_ep_combine(const CombineParams& p, int R, const int* rank_offsets,
                              const void* const* bufs, int64_t capacity_rows, void* y,
                              cudaStream_t stream) {
    if (p.T <= 0) return cudaSuccess;
    CombArgs a = comb_args(p, nullptr, y);
    a.rank_offsets = rank_offsets;
    a.ep_ranks = R;
    a.ep_capacity = capacity_rows;
    uintptr_t bits = (uintptr_t)p.row_bytes | reinterpret_cast<uintptr_t>(y);
    for (int r = 0; r < R; ++r) {
        a.ep_bufs[r] = bufs[r];
        bits |= reinterpret_cast<uintptr_t>(bufs[r]);
    }
    if (bits % 16 == 0) {
        a.rv = (int64_t)(p.row_bytes / 16);
        return launch_combine_k<uint4, MOE_COMBINE_VPL, true>(a, stream);
    }
    if (bits % 4 == 0) {
        a.rv = (int64_t)(p.row_bytes / 4);
        return launch_combine_k<uint32_t, 4, true>(a, stream);
    }
    a.rv = (int64_t)(p.row_bytes / 2);
    return launch_combine_k<uint16_t, 4, true>(a, stream);
}

cudaError_t launch_combine_rank_partials(const CombineParams& p, int R, const int* rank_offsets,
                                         const void* expert_out, float* partial,
                                         cudaStream_t stream) {
    if (p.T <= 0) return cudaSuccess;
    RankArgs ra;
    ra.c = comb_args(p, expert_out, nullptr);
    ra.R = R;
    ra.rank_offsets = rank_offsets;
    ra.partial = partial;
    const int vb = vec_bytes(p.row_bytes, expert_out, partial);
    auto go = [&](auto kern, int bytes) {
        ra.c.rv = (int64_t)(p.row_bytes / bytes);
        const int64_t cpr = (ra.c.rv + 31) / 32;
        int64_t g = ((int64_t)R * p.T * cpr + kWarpsPerCta - 1) / kWarpsPerCta;
        const int64_t cap = (int64_t)device_sm_count() * 16;
        return launch_pdl(kern, dim3((unsigned)(g > cap ? cap : g)), dim3(kThreads), 0, stream, ra);
    };
    if (vb == 16) return go(rank_partial_kernel<uint4>, 16);
    if (vb == 4) return go(rank_partial_kernel<uint32_t>, 4);
    return go(rank_partial_kernel<uint16_t>, 2);
}

cudaError_t launch_reduce_rank_partials(const CombineParams& p, int R, const float* partial,
                                        void* y, cudaStream_t stream) {
    if (p.T <= 0) return cudaSuccess;
    RankArgs ra;
    ra.c = comb_args(p, nullptr, y);
    ra.R = R;
    ra.rank_offsets = nullptr;
    ra.partial = const_cast<float*>(partial);
    const int vb = vec_bytes(p.row_bytes, partial, y);
    auto go = [&](auto kern, int bytes) {
        ra.c.rv = (int64_t)(p.row_bytes / bytes);
        return launch_pdl(kern, dim3((unsigned)(device_sm_count() * 8)), dim3(kThreads), 0, stream, ra);
    };
    if (vb == 16) return go(rank_reduce_kernel<uint4>, 16);
    if (vb == 4) return go(rank_reduce_kernel<uint32_t>, 4);
    return go(rank_reduce_kernel<uint16_t>, 2);
}

}  // namespace moe

// layout_common.cuh -- device helpers shared by the layout kernels
// (layout.cu) and the count + assign/dispatch kernels (fused.cu):
// reading one token's routes with the library's rule for invalid entries,
// and block / warp prefix scans.
#pragma once

#include "moe_common.cuh"

namespace moe {
namespace {

// Validate one token's k raw expert ids.  Invalid entries become -1 and set
// error bits: an id outside [0, E), or a repeat of an id earlier in the row
// (the later copy is dropped).  Every layout kernel uses this rule, so
// histograms and ranks always agree even on bad input.  Repeats are found
// with a 64-bit mask of ids seen so far (id mod 64); only when the mask hits
// are the earlier raw entries compared, which is exact because a valid id
// equal to an earlier raw id is a repeat.
template <int KMAX>
__device__ __forceinline__ int check_route(const int (&raw)[KMAX], int k, int E, int (&e)[KMAX]) {
    int bits = 0;
    uint64_t seen = 0;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        int v = -1;
        if (j < k) {
            v = raw[j];
            if (v < 0 || v >= E) {
                bits |= kErrExpertOob;
                v = -1;
            } else {
                const uint64_t bit = 1ull << (v & 63);
                if (seen & bit) {
                    bool repeat = false;
#pragma unroll
                    for (int i = 0; i < j; ++i) repeat |= raw[i] == v;
                    if (repeat) {
                        bits |= kErrDupExpert;
                        v = -1;
                    }
                }
                seen |= bit;
            }
        }
        e[j] = v;
    }
    return bits;
}

// Load token t's k expert ids from global memory (all k loads issued before
// any is examined, so they are in flight together) and validate them.
// vec4: k % 4 == 0 and topk 16-byte aligned, so the row is read as 16-byte
// vectors.
template <int KMAX>
__device__ __forceinline__ int load_route(const int* __restrict__ topk, int64_t t, int k, int E,
                                          int (&e)[KMAX], bool vec4 = false) {
    const int* row = topk + t * k;
    int raw[KMAX];
    if (vec4) {
#pragma unroll
        for (int q = 0; q < KMAX / 4; ++q) {
            int4 v = make_int4(-1, -1, -1, -1);
            if (4 * q < k) v = ld_dep4(row + 4 * q);
            raw[4 * q] = v.x;
            raw[4 * q + 1] = v.y;
            raw[4 * q + 2] = v.z;
            raw[4 * q + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < KMAX; ++j) raw[j] = j < k ? ld_dep(row + j) : -1;
    }
    return check_route<KMAX>(raw, k, E, e);
}

template <int KMAX>
__device__ __forceinline__ uint32_t node_mask(const Partition& part, const int (&e)[KMAX]) {
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
        if (e[j] >= 0) m |= 1u << part.node_of(e[j]);
    return m;
}

// The same from a shared-memory table of each expert's node (built once per
// CTA with fill_node_table), instead of two integer divisions per route.
template <int KMAX>
__device__ __forceinline__ uint32_t node_mask(const unsigned char* node_of, const int (&e)[KMAX]) {
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
        if (e[j] >= 0) m |= 1u << node_of[e[j]];
    return m;
}
__device__ __forceinline__ void fill_node_table(unsigned char* node_of, const Partition& part, int E) {
    for (int i = threadIdx.x; i < E; i += blockDim.x) node_of[i] = (unsigned char)part.node_of(i);
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

// In-place exclusive scan of an int array in shared memory (length L) by
// one block; returns the total.  s_warp holds 32 ints.
__device__ int smem_exclusive_scan(int* data, int L, int* s_warp) {
    const int span = (L + blockDim.x - 1) / blockDim.x;
    const int beg = min(L, (int)threadIdx.x * span);
    const int end = min(L, beg + span);
    int sum = 0;
    for (int i = beg; i < end; ++i) sum += data[i];
    int total = 0;
    int run = block_exclusive_scan(sum, s_warp, total);
    for (int i = beg; i < end; ++i) {
        const int v = data[i];
        data[i] = run;
        run += v;
    }
    __syncthreads();
    return total;
}

__device__ __forceinline__ int warp_inclusive_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFullMask, v, o);
        if (lane >= o) v += y;
    }
    return v;
}

}  // namespace
}  // namespace moe

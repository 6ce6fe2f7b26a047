// moe_common.cuh -- shared device helpers of the B200 MoE dispatch/combine
// kernels: error bits, the ceil/floor expert partition, cache-hinted vector
// loads/stores, bf16 packing and the launch wrapper.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <mutex>

namespace moe {

// Device error-word bits (moe_layout_t.error_word).
constexpr int kErrExpertOob = 1 << 0;
constexpr int kErrDupExpert = 1 << 1;
constexpr int kErrBadLayout = 1 << 2;
constexpr int kErrTimeout = 1 << 3;

constexpr unsigned kFullMask = 0xffffffffu;

// Ceil/floor contiguous expert partition (TensorRT-LLM PR #13888, PR
// description and the divisible-fast-path commit): base = E / R and rem =
// E % R are computed once; ranks below rem hold base + 1 experts.  When rem
// is zero the rank is a single division.
struct Partition {
    int E, R, base, rem, ranks_per_node;

    __host__ __device__ static Partition make(int E, int R, int N) {
        Partition p;
        p.E = E;
        p.R = R;
        p.base = E / R;
        p.rem = E % R;
        p.ranks_per_node = R / N;
        return p;
    }
    __host__ __device__ __forceinline__ int rank_of(int e) const {
        if (rem == 0) return e / base;
        const int big = rem * (base + 1);
        return e < big ? e / (base + 1) : rem + (e - big) / base;
    }
    __host__ __device__ __forceinline__ int first_expert(int r) const {
        return r * base + (r < rem ? r : rem);
    }
    __host__ __device__ __forceinline__ int node_of(int e) const {
        return rank_of(e) / ranks_per_node;
    }
};

// ---- programmatic dependent launch -------------------------------------
// Every kernel waits for its predecessor grid before touching memory and
// lets its dependent grid launch early, so launch latency overlaps the
// previous kernel's tail.
__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- cache-hinted global access -----------------------------------------
// Every kernel here may start before its predecessor on the stream has
// finished (programmatic dependent launch), so whatever a predecessor wrote
// (layout arrays, staging rows, receive rows, partial sums, scales) is read
// only after pdl_wait(), with coherent loads issued from volatile asm so that
// the compiler keeps them below the wait.  The non-coherent path
// (ld.global.nc, __ldg) is not used for such data: it assumes the data stays
// unchanged while the reading kernel is resident, and a reading kernel that
// is already resident while its predecessor writes breaks that assumption
// (the compiler may also hoist such a load above the wait).
__device__ __forceinline__ int ld_dep(const int* p) {
    int v;
    asm volatile("ld.global.s32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ int4 ld_dep4(const int* p) {  // 16-byte aligned
    int4 v;
    asm volatile("ld.global.v4.s32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ float ld_dep(const float* p) {
    float v;
    asm volatile("ld.global.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

// Streaming loads of rows read exactly once (no L1 allocation) and
// evict-first stores of rows written once.
template <typename V>
__device__ __forceinline__ V ld_stream(const V* p);
template <>
__device__ __forceinline__ uint4 ld_stream<uint4>(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
template <>
__device__ __forceinline__ uint2 ld_stream<uint2>(const uint2* p) {
    uint2 v;
    asm volatile("ld.global.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(v.x), "=r"(v.y)
                 : "l"(p));
    return v;
}
template <>
__device__ __forceinline__ uint32_t ld_stream<uint32_t>(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.global.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
template <>
__device__ __forceinline__ uint16_t ld_stream<uint16_t>(const uint16_t* p) {
    uint16_t v;
    asm volatile("ld.global.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

template <typename V>
__device__ __forceinline__ void st_stream(V* p, const V& v);
template <>
__device__ __forceinline__ void st_stream<uint4>(uint4* p, const uint4& v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}
template <>
__device__ __forceinline__ void st_stream<uint32_t>(uint32_t* p, const uint32_t& v) {
    asm volatile("st.global.cs.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
template <>
__device__ __forceinline__ void st_stream<uint16_t>(uint16_t* p, const uint16_t& v) {
    asm volatile("st.global.cs.u16 [%0], %1;" ::"l"(p), "h"(v) : "memory");
}

// ---- bf16 <-> fp32 over vector words -------------------------------------
// A bf16 value is the upper half of a binary32, so widening is a shift.
__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two fp32 -> two bf16 (round to nearest even, one cvt instruction).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&b);
}

// Number of bf16 values in one vector word.
template <typename V>
struct VecInfo;
template <>
struct VecInfo<uint4> {
    static constexpr int kElems = 8;
};
template <>
struct VecInfo<uint32_t> {
    static constexpr int kElems = 2;
};
template <>
struct VecInfo<uint16_t> {
    static constexpr int kElems = 1;
};

template <typename V>
__device__ __forceinline__ void unpack_bf16(const V& v, float (&f)[VecInfo<V>::kElems]);
template <>
__device__ __forceinline__ void unpack_bf16<uint4>(const uint4& v, float (&f)[8]) {
    f[0] = bf16lo_to_f32(v.x);
    f[1] = bf16hi_to_f32(v.x);
    f[2] = bf16lo_to_f32(v.y);
    f[3] = bf16hi_to_f32(v.y);
    f[4] = bf16lo_to_f32(v.z);
    f[5] = bf16hi_to_f32(v.z);
    f[6] = bf16lo_to_f32(v.w);
    f[7] = bf16hi_to_f32(v.w);
}
template <>
__device__ __forceinline__ void unpack_bf16<uint32_t>(const uint32_t& v, float (&f)[2]) {
    f[0] = bf16lo_to_f32(v);
    f[1] = bf16hi_to_f32(v);
}
template <>
__device__ __forceinline__ void unpack_bf16<uint16_t>(const uint16_t& v, float (&f)[1]) {
    f[0] = __uint_as_float(((uint32_t)v) << 16);
}

template <typename V>
__device__ __forceinline__ V pack_bf16(const float (&f)[VecInfo<V>::kElems]);
template <>
__device__ __forceinline__ uint4 pack_bf16<uint4>(const float (&f)[8]) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
}
template <>
__device__ __forceinline__ uint32_t pack_bf16<uint32_t>(const float (&f)[2]) {
    return pack_bf16x2(f[0], f[1]);
}
template <>
__device__ __forceinline__ uint16_t pack_bf16<uint16_t>(const float (&f)[1]) {
    __nv_bfloat16 b = __float2bfloat16_rn(f[0]);
    return *reinterpret_cast<uint16_t*>(&b);
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Record error bits once per warp.
__device__ __forceinline__ void warp_report(int* err_word, int bits) {
    const int any = __reduce_or_sync(kFullMask, bits);
    if (any && (threadIdx.x & 31) == 0 && err_word != nullptr) atomicOr(err_word, any);
}

// ---- per-CTA bulk copies (TMA, non-tensor) and mbarriers -------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
// Make mbarrier initialisation visible to the async (bulk copy) proxy.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}
// Bounded wait for an mbarrier phase: false once kMaxWaitNs of wall time
// (%globaltimer) have passed without the phase completing, which callers
// turn into kErrTimeout instead of spinning forever.  200 ms by default; a
// test build of the library shortens it with -DMOE_MAX_WAIT_NS=<ns>.
#ifndef MOE_MAX_WAIT_NS
#define MOE_MAX_WAIT_NS (200ull * 1000 * 1000)
#endif
constexpr uint64_t kMaxWaitNs = MOE_MAX_WAIT_NS;
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t start = global_ns();
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - start > kMaxWaitNs) return false;
    }
}
// global -> shared bulk copy completing on an mbarrier (bytes % 16 == 0,
// both addresses 16-byte aligned).
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// shared -> global bulk copy tracked by this thread's bulk groups.
__device__ __forceinline__ void bulk_store(void* gdst, const void* smem_src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
                 "r"(smem_u32(smem_src)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's committed groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until all of this thread's bulk groups have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ---- per-thread async copies (cp.async, global -> shared) -----------------
// Each thread tracks its own copies in commit groups; a copy's bytes may be
// read by the copying thread after cp.async.wait_group, by other threads of
// the warp after that and a __syncwarp().
__device__ __forceinline__ void async_copy16(void* smem_dst, const void* gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc)
                 : "memory");
}
__device__ __forceinline__ void async_copy4(void* smem_dst, const void* gsrc) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)), "l"(gsrc)
                 : "memory");
}
__device__ __forceinline__ void async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's committed groups are still pending.
template <int N>
__device__ __forceinline__ void async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---- launching ------------------------------------------------------------
// Launch with programmatic stream serialization allowed, so the kernel may
// start while its predecessor drains; each kernel calls pdl_wait() before
// it reads anything a predecessor wrote.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Streaming multiprocessors of the current device (cached per device).
int device_sm_count();

// Resident blocks per SM of a kernel at a block size and dynamic shared
// memory size, queried once per (kernel, threads, smem) and cached: a
// kernel's shared memory can depend on the row size (its chunk), so one
// process may launch it at several sizes.
template <auto Kernel>
inline int blocks_per_sm(int threads, size_t smem = 0) {
    struct Entry {
        int threads;
        size_t smem;
        int blocks;
    };
    constexpr int kSlots = 16;
    static Entry cache[kSlots] = {};
    static int used = 0;
    static std::mutex lock;
    std::lock_guard<std::mutex> guard(lock);
    for (int i = 0; i < used; ++i)
        if (cache[i].threads == threads && cache[i].smem == smem) return cache[i].blocks;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, Kernel, threads, smem) != cudaSuccess || n < 1) {
        cudaGetLastError();
        n = 1;
    }
    cache[used < kSlots ? used++ : kSlots - 1] = Entry{threads, smem, n};
    return n;
}

// Blocks of a kernel resident on the whole device at once.
template <auto Kernel>
inline int64_t resident_blocks(int threads, size_t smem = 0) {
    return (int64_t)device_sm_count() * blocks_per_sm<Kernel>(threads, smem);
}

// Where a row-moving kernel lets its dependent grid launch (programmatic
// dependent launch).  The dependent grid launches once every CTA of this
// grid has triggered or exited, and its CTAs then occupy SM slots while they
// wait for this grid to finish.  Triggering at entry hides the dependent's
// launch latency, which pays when the whole grid is resident at once.  In a
// grid of several waves, the entry trigger of the last wave lets the
// dependent's CTAs in while the last wave still moves rows, and measured on
// B200 that slowed the step (a one-kernel two-level dispatch followed by a
// combine: 809 us per step against 761 us with the trigger at the end).
// MOE_PDL_POLICY: 0 = always at entry, 1 = at the end for grids of more than
// one wave (default), 2 = always at the end.
#ifndef MOE_PDL_POLICY
#define MOE_PDL_POLICY 1
#endif
inline bool pdl_trigger_at_end(int64_t grid, int64_t resident) {
    if (MOE_PDL_POLICY == 0) return false;
    if (MOE_PDL_POLICY == 2) return true;
    return grid > resident;
}

// Grid for a warp-strided loop over `warp_items` items.  Small problems get
// a persistent grid (each warp one contiguous range of items).  When a
// resident grid would give each warp at least 2 * items_per_warp items, the
// grid becomes a whole number of resident waves (up to 16) of about
// items_per_warp items per warp: the block scheduler hands out the later
// waves as earlier blocks finish, so the kernel ends with every SM busy
// instead of a tail of slow warps, and no wave is left partly empty.
#ifndef MOE_ITEMS_PER_WARP
#define MOE_ITEMS_PER_WARP 4
#endif
constexpr int64_t kItemsPerWarp = MOE_ITEMS_PER_WARP;
template <auto Kernel>
inline int persistent_grid(int64_t warp_items, int threads, size_t smem = 0,
                           int64_t items_per_warp = kItemsPerWarp) {
    const int64_t warps_per_block = threads / 32;
    const int64_t resident = (int64_t)device_sm_count() * blocks_per_sm<Kernel>(threads, smem);
    int64_t g = (warp_items + warps_per_block - 1) / warps_per_block;   // one item per warp
    if (g > resident) {
        int64_t waves = warp_items / (resident * warps_per_block * items_per_warp);
        if (waves < 1) waves = 1;
        if (waves > 16) waves = 16;
        g = waves * resident;
    }
    return (int)(g < 1 ? 1 : g);
}

}  // namespace moe

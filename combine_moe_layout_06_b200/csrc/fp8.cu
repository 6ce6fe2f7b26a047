// fp8.cu -- fp8 (e4m3) payload for dispatch and combine.
//
// TensorRT-LLM PR #13888 (ConfigurableMoE commit) validates an fp8
// low-precision combine at rtol 0.02 / atol 0.15.  Rows travel as OCP E4M3
// codes with one fp32 scale per row: scale = amax / 448 (amax = the row's
// largest |value|; a zero row uses scale 1) and code = e4m3(v * (448 / amax)),
// rounded to nearest even and saturated to +-448 (cvt.rn.satfinite).  The
// receive buffer then carries H bytes plus 4 per row instead of 2H.
//
//  quantize_rows16_kernel (rows of up to 8192 values, H % 16 == 0): one
//    warp per source row, the row held in registers (lane l owns the
//    16-value groups l, l+32, ...), amax by a warp reduction, then every
//    group's 16 codes go out as one 16-byte store to every destination row:
//    the row itself (row-wise quantization of expert outputs) or the
//    token's k receive rows (fp8 dispatch: quantize once, write k copies).
//  quantize_fp8_kernel (any H % 8 == 0): the same with two passes over the
//    row (amax, then convert) and 8-byte code stores.
//  quantize_node_dispatch_kernel (two-level, H % 16 == 0, H <= 8192,
//    N + k <= 32): one warp per token quantizes its row once (row in
//    registers, as above), stores the codes and scale to the token's
//    staging row on every node it touches, then reads each staging row back
//    (from L2: the same lane's own bytes, ld.global.cg) and stores it to the
//    token's receive rows on that node.  The FUSCO article's forwarding
//    ("负载均衡与跨节点去重": a token crosses to a node once, then fans out
//    inside it) in one launch instead of a quantizer and two expansions.
//  combine_ring_fp8_kernel (H % 16 == 0, k <= 8) and combine_fp8_kernel
//    (any H % 8 == 0, k <= 32): the fused combine on codes, coef_j = w[t][j]
//    * scale[slot[t][j]] and acc = fma(coef_j, decode(code), acc) for j = 0
//    .. k-1 from +0, one RNE bf16 store.  The ring kernel stages the rows in
//    shared memory with cp.async, so more bytes are in flight per warp than
//    registers would hold; the code widening (e4m3 -> f16 -> f32 conversions)
//    then bounds it.
#include <cuda_fp8.h>

#include <climits>

#include "moe_kernels.h"

namespace moe {
namespace {

constexpr int kWarpsPerCta = 8;
constexpr int kThreads = kWarpsPerCta * 32;

// 8 floats -> 8 e4m3 codes (byte i = element i).
__device__ __forceinline__ uint2 to_e4m3x8(const float (&f)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        w[i] = (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(f[2 * i], f[2 * i + 1]), __NV_SATFINITE,
                                                  __NV_E4M3);
    return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

// 8 e4m3 codes -> 8 floats (exact): the hardware conversion of code pairs to
// f16x2, then each half widened to f32.
__device__ __forceinline__ void from_e4m3x8(uint2 c, float (&f)[8]) {
    const uint32_t w[2] = {c.x, c.y};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)(w[i >> 1] >> (16 * (i & 1)));
        const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
        f[2 * i] = __half2float(__half(__half_raw{h.x}));
        f[2 * i + 1] = __half2float(__half(__half_raw{h.y}));
    }
}

struct Fp8Args {
    const uint4* src;     // bf16 rows, 8 values per vector
    uint2* q;             // e4m3 rows, 8 codes per vector
    float* scale;         // one per destination row
    const int* slot;      // nullptr: the destination of row r is row r
    const int* dst_base;  // nullptr, or per-column first rows (node staging)
    int64_t rows;         // source rows
    int k;                // destinations per source row (slot mode)
    int64_t rv;           // vectors per row (H / 8)
    int64_t dst_rows;
    int* err;
};

// Lane j's destination row of source row r (-1: none): row r itself, or
// dst_base[j] + slot[r][j] for j < k (a receive row, or a node's staging row).
__device__ __forceinline__ int64_t quant_dst(const Fp8Args& a, int64_t r, int lane, int& errbits) {
    if (a.slot == nullptr) return lane == 0 ? r : -1;
    if (lane >= a.k) return -1;
    const int s = ld_dep(a.slot + r * a.k + lane);
    if (s < 0) {
        if (s != -1) errbits |= kErrBadLayout;
        return -1;
    }
    const int64_t d = (a.dst_base ? (int64_t)ld_dep(a.dst_base + lane) : 0) + s;
    if (d < a.dst_rows) return d;
    errbits |= kErrBadLayout;
    return -1;
}

__global__ void __launch_bounds__(kThreads) quantize_fp8_kernel(Fp8Args a) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t nw = (int64_t)gridDim.x * kWarpsPerCta;
    int errbits = 0;
    for (int64_t r = (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5); r < a.rows; r += nw) {
        const int64_t dst = quant_dst(a, r, lane, errbits);
        const uint4* src = a.src + r * a.rv;
        uint32_t amax_bits = 0;
        for (int64_t v = lane; v < a.rv; v += 32) {
            float f[8];
            unpack_bf16<uint4>(ld_stream(src + v), f);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const uint32_t b = __float_as_uint(fabsf(f[e]));
                if (b <= 0x7F800000u) amax_bits = max(amax_bits, b);   // NaNs have no magnitude
            }
        }
        amax_bits = __reduce_max_sync(kFullMask, amax_bits);
        const float amax = __uint_as_float(amax_bits);
        const float inv = amax > 0.f ? 448.0f / amax : 1.0f;
        const float scale = amax > 0.f ? amax / 448.0f : 1.0f;
        const unsigned dmask = __ballot_sync(kFullMask, dst >= 0);
        if (dst >= 0) a.scale[dst] = scale;
        // every lane runs every pass (the destination shuffles need the warp)
        for (int64_t v0 = 0; v0 < a.rv; v0 += 32) {
            const int64_t v = v0 + lane;
            const bool active = v < a.rv;
            float f[8];
            uint4 raw = make_uint4(0, 0, 0, 0);
            if (active) raw = ld_stream(src + v);
            unpack_bf16<uint4>(raw, f);
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = f[e] * inv;
            const uint2 code = to_e4m3x8(f);
            unsigned m = dmask;
            while (m) {
                const int j = __ffs(m) - 1;
                m &= m - 1;
                const int64_t d = __shfl_sync(kFullMask, dst, j);
                if (active) a.q[d * a.rv + v] = code;
            }
        }
    }
    warp_report(a.err, errbits);
}

// Register-resident row: NG 16-value groups per lane (H <= 512 * NG), W
// warps per CTA.  Codes are made one group at a time and stored to every
// destination at once, so only the raw row stays in registers.
template <int NG, int W>
__global__ void __launch_bounds__(W * 32) quantize_rows16_kernel(Fp8Args a) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t G = a.rv / 2;  // 16-value groups per row
    const int64_t nw = (int64_t)gridDim.x * W;
    int errbits = 0;
    for (int64_t r = (int64_t)blockIdx.x * W + (threadIdx.x >> 5); r < a.rows; r += nw) {
        const int64_t dst = quant_dst(a, r, lane, errbits);
        const uint4* src = a.src + r * a.rv;
        uint4 raw[NG][2];
#pragma unroll
        for (int i = 0; i < NG; ++i) {
            const int64_t g = lane + 32 * i;
            raw[i][0] = raw[i][1] = make_uint4(0, 0, 0, 0);
            if (g < G) {
                raw[i][0] = ld_stream(src + 2 * g);
                raw[i][1] = ld_stream(src + 2 * g + 1);
            }
        }
        // |v| of a bf16 orders like its low 15 bits (infinity above every
        // finite value): a per-halfword integer max finds amax's bits; NaNs
        // (above 0x7F80) have no magnitude and are masked out
        uint32_t m2 = 0;
        auto fold = [&](uint32_t w) {
            const uint32_t x = w & 0x7FFF7FFFu;
            m2 = __vmaxu2(m2, x & ~__vcmpgtu2(x, 0x7F807F80u));
        };
#pragma unroll
        for (int i = 0; i < NG; ++i)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                fold(raw[i][h].x);
                fold(raw[i][h].y);
                fold(raw[i][h].z);
                fold(raw[i][h].w);
            }
        uint32_t amax_bits = max(m2 & 0xFFFFu, m2 >> 16) << 16;
        amax_bits = __reduce_max_sync(kFullMask, amax_bits);
        const float amax = __uint_as_float(amax_bits);
        const float inv = amax > 0.f ? 448.0f / amax : 1.0f;
        const float scale = amax > 0.f ? amax / 448.0f : 1.0f;
        if (dst >= 0) a.scale[dst] = scale;
        const unsigned dmask = __ballot_sync(kFullMask, dst >= 0);
        uint4* q = reinterpret_cast<uint4*>(a.q);
#pragma unroll
        for (int i = 0; i < NG; ++i) {
            uint2 c[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float f[8];
                unpack_bf16<uint4>(raw[i][h], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = f[e] * inv;
                c[h] = to_e4m3x8(f);
            }
            const uint4 code = make_uint4(c[0].x, c[0].y, c[1].x, c[1].y);
            const int64_t g = lane + 32 * i;
            unsigned m = dmask;
            while (m) {
                const int j = __ffs(m) - 1;
                m &= m - 1;
                const int64_t d = __shfl_sync(kFullMask, dst, j);
                if (g < G) st_stream(q + d * G + g, code);
            }
        }
    }
    warp_report(a.err, errbits);
}

// One-kernel fp8 two-level dispatch (see the file comment).
struct Fp8NodeArgs {
    const uint4* src;        // bf16 x rows, 8 values per vector
    int64_t T;
    int k, N, ranks_per_node;
    int64_t G;               // 16-value groups per row
    const int* slot;         // [T*k]
    const int* node_slot;    // [T*N]
    const int* node_offsets; // [N+1]
    const int* rank_offsets; // [R+1]
    uint4* staging_q;        // [staging_rows][G] 16-code groups
    float* staging_s;
    int64_t staging_rows;
    uint4* recv_q;           // [recv_rows][G]
    float* recv_s;
    int64_t recv_rows;
    int* err;
    int late_trigger;        // let the dependent grid launch at the end (pdl_trigger_at_end)
};

__device__ __forceinline__ uint4 ld_l2(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ float ld_l2(const float* p) {
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

// 32 contiguous bytes per lane in one access (sm_100's 256-bit loads and
// stores); p 32-byte aligned.
__device__ __forceinline__ void ld_stream_pair(const uint4* p, uint4& u, uint4& v) {
    asm volatile("ld.global.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w), "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
}
__device__ __forceinline__ void ld_l2_pair(const uint4* p, uint4& u, uint4& v) {
    asm volatile("ld.global.cg.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w), "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
}
__device__ __forceinline__ void st_pair(uint4* p, const uint4& u, const uint4& v) {
    asm volatile("st.global.v8.u32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(u.x), "r"(u.y),
                 "r"(u.z), "r"(u.w), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ void st_stream_pair(uint4* p, const uint4& u, const uint4& v) {
    asm volatile("st.global.cs.v8.u32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(u.x), "r"(u.y),
                 "r"(u.z), "r"(u.w), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// PAIR (G even; x, staging and receive codes 32-byte aligned): lane l owns
// the 16-value groups 2l + 64p and 2l + 64p + 1 (p < NG/2) instead of l + 32i,
// so its two groups' codes are 32 contiguous bytes and every load, store and
// read-back is one 32-byte access: half the load/store-queue entries of the
// 16-byte form.
template <int NG, int W, bool PAIR = false>
__global__ void __launch_bounds__(W * 32) quantize_node_dispatch_kernel(Fp8NodeArgs a) {
    static_assert(!PAIR || NG % 2 == 0, "paired groups");
    constexpr int kStep = PAIR ? 2 : 1;  // groups handled per access
    constexpr int kNext = PAIR ? 1 : 0;  // offset of the second group of an access
    // lane's i-th 16-value group
    auto grp = [](int i) -> int64_t {
        const int l = threadIdx.x & 31;
        return PAIR ? 2 * l + 64 * (i >> 1) + (i & 1) : l + 32 * i;
    };
    if (!a.late_trigger) pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int N = a.N;
    // node n: lane n holds its receive-row range [lo, hi); lane 31 - n its
    // first staging row
    int n_lo = INT_MAX, n_hi = INT_MIN, n_first = 0;
    if (lane < N) {
        n_lo = ld_dep(a.rank_offsets + lane * a.ranks_per_node);
        n_hi = ld_dep(a.rank_offsets + (lane + 1) * a.ranks_per_node);
    }
    const bool stager = lane >= 32 - N;
    const int my_node = 31 - lane;
    if (stager) n_first = ld_dep(a.node_offsets + my_node);
    const int64_t G = a.G;
    const int64_t nw = (int64_t)gridDim.x * W;
    int errbits = 0;
    for (int64_t t = (int64_t)blockIdx.x * W + (threadIdx.x >> 5); t < a.T; t += nw) {
        // column j's receive row and its node; node n's staging row
        int sl = -1, nj = -1;
        int64_t srow = -1;
        if (lane < a.k) {
            const int s = ld_dep(a.slot + t * a.k + lane);
            if (s >= 0 && s < a.recv_rows) sl = s;
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
        // the row, held in registers: lane l owns 16-value groups l, l+32, ...
        const uint4* src = a.src + t * 2 * G;
        uint4 raw[NG][2];
#pragma unroll
        for (int i = 0; i < NG; ++i) {
            const int64_t g = grp(i);
            raw[i][0] = raw[i][1] = make_uint4(0, 0, 0, 0);
            if (g < G) {
                if (PAIR) {
                    ld_stream_pair(src + 2 * g, raw[i][0], raw[i][1]);
                } else {
                    raw[i][0] = ld_stream(src + 2 * g);
                    raw[i][1] = ld_stream(src + 2 * g + 1);
                }
            }
        }
        // amax as quantize_rows16_kernel finds it (NaNs have no magnitude)
        uint32_t m2 = 0;
        auto fold = [&](uint32_t w) {
            const uint32_t x = w & 0x7FFF7FFFu;
            m2 = __vmaxu2(m2, x & ~__vcmpgtu2(x, 0x7F807F80u));
        };
#pragma unroll
        for (int i = 0; i < NG; ++i)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                fold(raw[i][h].x);
                fold(raw[i][h].y);
                fold(raw[i][h].z);
                fold(raw[i][h].w);
            }
        uint32_t amax_bits = max(m2 & 0xFFFFu, m2 >> 16) << 16;
        amax_bits = __reduce_max_sync(kFullMask, amax_bits);
        const float amax = __uint_as_float(amax_bits);
        const float inv = amax > 0.f ? 448.0f / amax : 1.0f;
        const float scale = amax > 0.f ? amax / 448.0f : 1.0f;
        // 1. codes and scale into the staging row of every node touched
        if (srow >= 0) a.staging_s[srow] = scale;
        const unsigned smask = __ballot_sync(kFullMask, srow >= 0);  // bit 31 - n: node n
        auto quantize = [&](int i) {
            uint2 c[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float f[8];
                unpack_bf16<uint4>(raw[i][h], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = f[e] * inv;
                c[h] = to_e4m3x8(f);
            }
            return make_uint4(c[0].x, c[0].y, c[1].x, c[1].y);
        };
#pragma unroll
        for (int i = 0; i < NG; i += kStep) {
            const uint4 code = quantize(i);
            const uint4 code2 = PAIR ? quantize(i + kNext) : code;
            const int64_t g = grp(i);
            unsigned m = smask;
            while (m) {
                const int j = __ffs(m) - 1;
                m &= m - 1;
                const int64_t d = __shfl_sync(kFullMask, srow, j);
                if (g < G) {
                    if (PAIR) st_pair(a.staging_q + d * G + g, code, code2);
                    else a.staging_q[d * G + g] = code;
                }
            }
        }
        __syncwarp();  // the staging scales are seen by the lanes that read them back
        // 2. each staging row read back and stored to the node's receive rows
        unsigned m = smask;
        while (m) {
            const int j = __ffs(m) - 1;
            m &= m - 1;
            const int n = 31 - j;
            const int64_t row_n = __shfl_sync(kFullMask, srow, j);
            const unsigned cols = __ballot_sync(kFullMask, sl >= 0 && nj == n);
            if ((cols >> lane) & 1u) a.recv_s[sl] = ld_l2(a.staging_s + row_n);
            uint4 back[NG];
#pragma unroll
            for (int i = 0; i < NG; i += kStep) {
                const int64_t g = grp(i);
                back[i] = back[i + kNext] = make_uint4(0, 0, 0, 0);
                if (g < G) {
                    if (PAIR) ld_l2_pair(a.staging_q + row_n * G + g, back[i], back[i + kNext]);
                    else back[i] = ld_l2(a.staging_q + row_n * G + g);
                }
            }
            unsigned cm = cols;
            while (cm) {
                const int q = __ffs(cm) - 1;
                cm &= cm - 1;
                const int64_t d = __shfl_sync(kFullMask, (int64_t)sl, q);
#pragma unroll
                for (int i = 0; i < NG; i += kStep) {
                    const int64_t g = grp(i);
                    if (g < G) {
                        if (PAIR) st_stream_pair(a.recv_q + d * G + g, back[i], back[i + kNext]);
                        else st_stream(a.recv_q + d * G + g, back[i]);
                    }
                }
            }
        }
    }
    if (a.late_trigger) pdl_trigger();
    warp_report(a.err, errbits);
}

struct Fp8CombArgs {
    const uint2* q;        // e4m3 expert rows
    const float* scale;    // per expert row
    const float* w;        // [T*k]
    const int* slot;       // [T*k]
    uint4* y;              // bf16 rows
    int64_t T;
    int k;
    int64_t rv;            // 8-value vectors per row
    int64_t q_rows;
    int* err;
};

// Items are (token, chunk of 32*VPL vectors), a contiguous token-major range
// per warp; lanes hold the token's slots and coefficients; up to 8 rows'
// codes are loaded before their FMAs.
template <int VPL>
__global__ void __launch_bounds__(kThreads) combine_fp8_kernel(Fp8CombArgs a) {
    constexpr int CHUNK = 32 * VPL;
    constexpr int KB = 8;
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t cpr = (a.rv + CHUNK - 1) / CHUNK;
    const int64_t items = a.T * cpr;
    const int64_t nw = (int64_t)gridDim.x * kWarpsPerCta;
    const int64_t gw = (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    const int64_t ib = items * gw / nw, ie = items * (gw + 1) / nw;
    int errbits = 0;
    int64_t t_loaded = -1;
    int s = -1;
    float coef = 0.f;
    for (int64_t item = ib; item < ie; ++item) {
        const int64_t t = item / cpr;
        const int64_t base = (item - t * cpr) * CHUNK;
        if (t != t_loaded) {
            s = -1;
            coef = 0.f;
            if (lane < a.k) {
                s = ld_dep(a.slot + t * a.k + lane);
                if (s >= 0 && s < a.q_rows) coef = ld_dep(a.w + t * a.k + lane) * ld_dep(a.scale + s);
                else {
                    if (s != -1) errbits |= kErrBadLayout;
                    s = -1;
                }
            }
            t_loaded = t;
        }
        float acc[VPL][8];
#pragma unroll
        for (int i = 0; i < VPL; ++i)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[i][e] = 0.f;
        for (int j0 = 0; j0 < a.k; j0 += KB) {
            uint2 v[KB][VPL];
            float cq[KB];
            bool ok[KB];
#pragma unroll
            for (int q = 0; q < KB; ++q) {
                const int j = j0 + q;
                const int sj = __shfl_sync(kFullMask, s, j & 31);
                cq[q] = __shfl_sync(kFullMask, coef, j & 31);
                ok[q] = j < a.k && sj >= 0;
                if (ok[q]) {
#pragma unroll
                    for (int i = 0; i < VPL; ++i) {
                        const int64_t idx = base + i * 32 + lane;
                        if (idx < a.rv) v[q][i] = ld_stream(a.q + (int64_t)sj * a.rv + idx);
                    }
                }
            }
#pragma unroll
            for (int q = 0; q < KB; ++q) {
                if (!ok[q]) continue;
#pragma unroll
                for (int i = 0; i < VPL; ++i) {
                    if (base + i * 32 + lane < a.rv) {
                        float f[8];
                        from_e4m3x8(v[q][i], f);
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[i][e] = __fmaf_rn(cq[q], f[e], acc[i][e]);
                    }
                }
            }
        }
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int64_t idx = base + i * 32 + lane;
            if (idx < a.rv) a.y[t * a.rv + idx] = pack_bf16<uint4>(acc[i]);
        }
    }
    warp_report(a.err, errbits);
}

// Shared-memory staged combine (H % 16 == 0, k <= 8): each warp keeps a
// ring of kRing stages, a stage holding one item's (token, 512-code chunk)
// rows -- lane l copies group l of every expert row with cp.async -- plus
// the rows' weights and scales.  The data in flight lives in shared memory,
// not registers, so kRing - 1 items per warp stay in flight while one is
// summed.  Items are a contiguous token-major range per warp; rows are
// summed in column order j = 0 .. k-1 exactly as in the register kernels.
#ifndef MOE_FP8_RING
#define MOE_FP8_RING 3
#endif
#ifndef MOE_FP8_RING_WARPS
#define MOE_FP8_RING_WARPS 8
#endif
constexpr int kRing = MOE_FP8_RING;
constexpr int kRingWarps = MOE_FP8_RING_WARPS;
constexpr int kRingThreads = kRingWarps * 32;
constexpr int kRingRows = 8;
struct RingStage {
    uint4 code[kRingRows][32];  // [row j][lane]
    float w[kRingRows];
    float scale[kRingRows];
    unsigned valid;             // bit j: row j is summed
    unsigned pad[3];
};

__global__ void __launch_bounds__(kRingThreads) combine_ring_fp8_kernel(Fp8CombArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    RingStage* ring = reinterpret_cast<RingStage*>(smem) + warp * kRing;
    pdl_trigger();
    pdl_wait();
    const int64_t G = a.rv / 2;   // 16-code groups per row
    const int64_t cpr = (G + 31) / 32;
    const int64_t items = a.T * cpr;
    const int64_t nw = (int64_t)gridDim.x * kRingWarps;
    const int64_t gw = (int64_t)blockIdx.x * kRingWarps + warp;
    const int64_t ib = items * gw / nw, ie = items * (gw + 1) / nw;
    const uint4* q = reinterpret_cast<const uint4*>(a.q);
    int errbits = 0;

    // issue side: lane j < k holds the expert row of (token ti, j)
    int64_t ti = -1;
    int s_issue = -1;
    auto issue = [&](int64_t item, RingStage& st) {
        const int64_t t = item / cpr;
        const int64_t g = (item - t * cpr) * 32 + lane;
        if (t != ti) {
            s_issue = -1;
            if (lane < a.k) {
                const int s = ld_dep(a.slot + t * a.k + lane);
                if (s >= 0 && s < a.q_rows) s_issue = s;
                else if (s != -1) errbits |= kErrBadLayout;
            }
            ti = t;
        }
        const unsigned valid = __ballot_sync(kFullMask, s_issue >= 0);
        if (lane == 0) st.valid = valid;
        if (s_issue >= 0) {
            async_copy4(&st.w[lane], a.w + t * a.k + lane);
            async_copy4(&st.scale[lane], a.scale + s_issue);
        }
        unsigned m = valid;
        while (m) {
            const int j = __ffs(m) - 1;
            m &= m - 1;
            const int sj = __shfl_sync(kFullMask, s_issue, j);
            if (g < G) async_copy16(&st.code[j][lane], q + (int64_t)sj * G + g);
        }
        async_commit();
    };

    const int64_t mine = ie - ib;
    for (int64_t i = 0; i < kRing - 1; ++i) {
        if (i < mine) issue(ib + i, ring[i]);
        else async_commit();   // keep one group per stage
    }
    for (int64_t i = 0; i < mine; ++i) {
        // refill the stage freed last iteration, then wait for item i
        if (i + kRing - 1 < mine) issue(ib + i + kRing - 1, ring[(i + kRing - 1) % kRing]);
        else async_commit();
        async_wait<kRing - 1>();
        __syncwarp();
        RingStage& st = ring[i % kRing];
        const int64_t item = ib + i;
        const int64_t t = item / cpr;
        const int64_t g = (item - t * cpr) * 32 + lane;
        const unsigned valid = st.valid;
        float acc[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] = 0.f;
#pragma unroll
        for (int j = 0; j < kRingRows; ++j) {
            if (!((valid >> j) & 1u)) continue;
            const float coef = st.w[j] * st.scale[j];
            const uint4 c = st.code[j][lane];
            float f[8];
            from_e4m3x8(make_uint2(c.x, c.y), f);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = __fmaf_rn(coef, f[e], acc[e]);
            from_e4m3x8(make_uint2(c.z, c.w), f);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[8 + e] = __fmaf_rn(coef, f[e], acc[8 + e]);
        }
        if (g < G) {
            float lo[8], hi[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                lo[e] = acc[e];
                hi[e] = acc[8 + e];
            }
            uint4* yrow = a.y + t * a.rv;
            st_stream(yrow + 2 * g, pack_bf16<uint4>(lo));
            st_stream(yrow + 2 * g + 1, pack_bf16<uint4>(hi));
        }
        // every lane has read this stage before it is refilled
        __syncwarp();
    }
    async_wait<0>();
    warp_report(a.err, errbits);
}

}  // namespace

bool fp8_eligible(int64_t hidden, std::initializer_list<const void*> bf16_ptrs,
                  std::initializer_list<const void*> q_ptrs) {
    if (hidden % 8 != 0) return false;
    for (const void* p : bf16_ptrs)
        if (reinterpret_cast<uintptr_t>(p) % 16) return false;
    for (const void* p : q_ptrs)
        if (reinterpret_cast<uintptr_t>(p) % 8) return false;
    return true;
}

namespace {
template <int NG, int W>
cudaError_t launch_rows16(const Fp8Args& a, cudaStream_t stream) {
    constexpr auto kern = quantize_rows16_kernel<NG, W>;
    const int grid = persistent_grid<kern>(a.rows, W * 32);
    return launch_pdl(kern, dim3(grid), dim3(W * 32), 0, stream, a);
}
}  // namespace

cudaError_t launch_quantize_fp8(const void* src, int64_t rows, int64_t hidden, const int* slot, int k,
                                int64_t dst_rows, void* q, float* scale, int* err,
                                cudaStream_t stream, const int* dst_base) {
    if (rows <= 0) return cudaSuccess;
    Fp8Args a;
    a.src = static_cast<const uint4*>(src);
    a.q = static_cast<uint2*>(q);
    a.scale = scale;
    a.slot = slot;
    a.dst_base = dst_base;
    a.rows = rows;
    a.k = k;
    a.rv = hidden / 8;
    a.dst_rows = dst_rows;
    a.err = err;
    // register-resident rows when the row splits into 16-value groups, at
    // most 8 per lane, and the codes take 16-byte stores
    const bool wide = hidden % 16 == 0 && reinterpret_cast<uintptr_t>(q) % 16 == 0;
    if (wide && hidden <= 512 * 2) return launch_rows16<2, 8>(a, stream);
    if (wide && hidden <= 512 * 4) return launch_rows16<4, 8>(a, stream);
    if (wide && hidden <= 512 * 8) return launch_rows16<8, 8>(a, stream);
    if (wide && hidden <= 512 * 16) return launch_rows16<16, 4>(a, stream);
    constexpr auto kern = quantize_fp8_kernel;
    const int grid = persistent_grid<kern>(rows, kThreads);
    return launch_pdl(kern, dim3(grid), dim3(kThreads), 0, stream, a);
}

namespace {
template <int NG, int W, bool PAIR>
cudaError_t launch_node_q_form(Fp8NodeArgs a, cudaStream_t stream) {
    constexpr auto kern = quantize_node_dispatch_kernel<NG, W, PAIR>;
    const int grid = persistent_grid<kern>(a.T, W * 32);
    a.late_trigger = pdl_trigger_at_end(grid, resident_blocks<kern>(W * 32)) ? 1 : 0;
    return launch_pdl(kern, dim3(grid), dim3(W * 32), 0, stream, a);
}
// The paired (32-byte) form where the groups pair up and the buffers allow
// it (compile-time switch MOE_FP8_NODE_PAIR; 0 = never).
#ifndef MOE_FP8_NODE_PAIR
#define MOE_FP8_NODE_PAIR 1
#endif
template <int NG, int W>
cudaError_t launch_node_q(Fp8NodeArgs a, cudaStream_t stream) {
    const uintptr_t align = reinterpret_cast<uintptr_t>(a.src) | reinterpret_cast<uintptr_t>(a.staging_q) |
                            reinterpret_cast<uintptr_t>(a.recv_q);
    if (MOE_FP8_NODE_PAIR && a.G % 2 == 0 && align % 32 == 0) return launch_node_q_form<NG, W, true>(a, stream);
    return launch_node_q_form<NG, W, false>(a, stream);
}
}  // namespace

bool fp8_node_dispatch_eligible(const RowMoveParams& p, int64_t hidden, std::initializer_list<const void*> ptrs) {
    uintptr_t bits = 0;
    for (const void* q : ptrs) bits |= reinterpret_cast<uintptr_t>(q);
    return hidden % 16 == 0 && hidden <= 512 * 16 && p.N + p.k <= 32 && bits % 16 == 0;
}

cudaError_t launch_fp8_node_dispatch(const RowMoveParams& p, const void* x, int64_t hidden,
                                     void* staging_q, float* staging_scale, int64_t staging_rows,
                                     void* recv_q, float* recv_scale, cudaStream_t stream) {
    if (p.T <= 0) return cudaSuccess;
    Fp8NodeArgs a;
    a.src = static_cast<const uint4*>(x);
    a.T = p.T;
    a.k = p.k;
    a.N = p.N;
    a.ranks_per_node = p.ranks_per_node;
    a.G = hidden / 16;
    a.slot = p.slot;
    a.node_slot = p.node_slot;
    a.node_offsets = p.node_offsets;
    a.rank_offsets = p.rank_offsets;
    a.staging_q = static_cast<uint4*>(staging_q);
    a.staging_s = staging_scale;
    a.staging_rows = staging_rows;
    a.recv_q = static_cast<uint4*>(recv_q);
    a.recv_s = recv_scale;
    a.recv_rows = p.T * p.k;
    a.err = p.err;
    a.late_trigger = 0;
    if (hidden <= 512 * 2) return launch_node_q<2, 8>(a, stream);
    if (hidden <= 512 * 4) return launch_node_q<4, 8>(a, stream);
    if (hidden <= 512 * 8) return launch_node_q<8, 8>(a, stream);
    return launch_node_q<16, 4>(a, stream);
}

cudaError_t launch_combine_fp8(const CombineParams& p, const void* q, const float* scale, void* y,
                               cudaStream_t stream) {
    if (p.T <= 0) return cudaSuccess;
    Fp8CombArgs a;
    a.q = static_cast<const uint2*>(q);
    a.scale = scale;
    a.w = p.w;
    a.slot = p.slot;
    a.y = static_cast<uint4*>(y);
    a.T = p.T;
    a.k = p.k;
    a.rv = (int64_t)(p.row_bytes / 16);
    a.q_rows = p.T * p.k;
    a.err = p.err;
    const bool wide = (p.row_bytes / 2) % 16 == 0 && reinterpret_cast<uintptr_t>(q) % 16 == 0;
    if (wide && p.k <= kRingRows) {
        constexpr auto kr = combine_ring_fp8_kernel;
        const size_t smem = sizeof(RingStage) * kRing * kRingWarps;
        cudaError_t e = cudaFuncSetAttribute(kr, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const int64_t cprr = (a.rv / 2 + 31) / 32;
        const int gridr = persistent_grid<kr>(a.T * cprr, kRingThreads, smem);
        return launch_pdl(kr, dim3(gridr), dim3(kRingThreads), smem, stream, a);
    }
    constexpr auto kern = combine_fp8_kernel<2>;
    const int64_t cpr = (a.rv + 63) / 64;
    const int grid = persistent_grid<kern>(a.T * cpr, kThreads);
    return launch_pdl(kern, dim3(grid), dim3(kThreads), 0, stream, a);
}

}  // namespace moe

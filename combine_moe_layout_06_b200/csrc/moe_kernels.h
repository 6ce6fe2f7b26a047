// moe_kernels.h -- host launchers of the MoE dispatch/combine kernels
// (internal to libmoe_layout.so; the public C ABI is include/moe_layout.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include <initializer_list>
#include <stdint.h>

#include "moe_common.cuh"

namespace moe {

// Which row-copy engine moves bf16 rows.
enum class CopyEngine { kAuto = 0, kVector = 1, kBulk = 2 };

// ---- layout ----------------------------------------------------------------
struct LayoutParams {
    int64_t T;
    int k, E, R, N;
    bool nodes;             // also build node staging maps
    bool cluster;           // single cluster launch (T <= 131072)
    const int* topk;        // [T*k]
    int* expert_counts;     // [E]
    int* expert_offsets;    // [E+1]
    int* rank_offsets;      // [R+1]
    int* slot;              // [T*k]
    int* node_counts;       // [N]    (nodes)
    int* node_offsets;      // [N+1]  (nodes)
    int* node_slot;         // [T*N]  (nodes)
    int* node_src = nullptr;  // [U]  staging row -> token (nodes, optional)
    int* err;               // [1]
    void* workspace;        // layout_workspace_bytes()
};
// Workspace bytes: the layout kernels' chunk histograms and, for flat
// layouts (no node maps), the region of the count + assign/dispatch pair
// (fused.cu) after them: kFusedBarrierBytes holding a ticket counter, which
// must be zero before the first launch and is left zero by every launch,
// then an [E][kFusedMaxCtas] histogram matrix.
size_t layout_workspace_bytes(int64_t T, int E, int N, bool nodes);
// The part of the workspace launch_layout() itself reads and writes (the
// chunk histograms, and the node histograms with node staging); every word
// of it is written by a launch before that launch reads it.
size_t layout_scratch_bytes(int64_t T, int E, int N, bool nodes);
cudaError_t launch_layout(const LayoutParams& p, cudaStream_t stream);

// ---- layout and flat dispatch, assignment folded into the dispatch (fused.cu)
constexpr int kFusedMaxCtas = 256;      // columns of the histogram matrix
constexpr int kFusedMaxExperts = 256;   // shared-memory lane masks per expert
constexpr int kFusedMaxTopk = 32;
constexpr size_t kFusedBarrierBytes = 256;
// Byte offset of the fused region inside the workspace (flat layouts).
size_t fused_workspace_offset(int64_t T, int E);
// Whether the count + assign/dispatch pair takes this problem (16-byte
// aligned rows are checked by the caller).
bool layout_dispatch_fused_eligible(int64_t T, int k, int E, size_t row_bytes);
// moe_layout() (flat) + moe_dispatch() as the count + assign/dispatch pair;
// lp.nodes must be false and lp.workspace must hold layout_workspace_bytes().
cudaError_t launch_layout_dispatch_fused(const LayoutParams& lp, const void* x, void* recv,
                                         size_t row_bytes, cudaStream_t stream);

// ---- row movement ------------------------------------------------------------
// Geometry shared by the dispatch-side kernels.  Row sizes are in bytes;
// every row of x / recv / staging is row_bytes long and rows are packed.
struct RowMoveParams {
    int64_t T;
    int k, N, ranks_per_node;
    size_t row_bytes;
    const int* slot;          // [T*k]
    const int* node_slot;     // [T*N]
    const int* node_offsets;  // [N+1]
    const int* rank_offsets;  // [R+1]
    // [U] staging row -> token; when given, the node expansion walks staging
    // rows (work divided by rows, whatever each node's load), else (node,
    // token) pairs
    const int* node_src = nullptr;
    int* err;
    CopyEngine engine;
    // The source rows (x) were complete before the layout began and the
    // kernel runs right behind the layout kernels: the bulk engine may start
    // loading source rows before waiting for the layout.
    bool early_inputs = false;
};

// recv[slot[t][j]] = x[t]
cudaError_t launch_dispatch_flat(const RowMoveParams& p, const void* x, void* recv,
                                 cudaStream_t stream);
// staging[node_offsets[n] + node_slot[t][n]] = x[t] for every node touched
cudaError_t launch_node_pack(const RowMoveParams& p, const void* x, void* staging,
                             int64_t staging_rows, cudaStream_t stream);
// recv[slot[t][j]] = staging[node row of (t, n)] for the j whose row lies on n
cudaError_t launch_node_expand(const RowMoveParams& p, const void* staging,
                               int64_t staging_rows, void* recv, cudaStream_t stream);
// dst[0 .. rows) = src[0 .. rows); rows = *rows_dev (clamped to max_rows)
// when rows_dev is given, else max_rows.
cudaError_t launch_copy_rows(const void* src, void* dst, const int* rows_dev, int64_t max_rows,
                             size_t row_bytes, cudaStream_t stream);
// gathered[r*T + t] = x[t] for r < p.N (p.N = rank count; all-gather)
cudaError_t launch_allgather_rows(const RowMoveParams& p, const void* x, void* gathered,
                                  cudaStream_t stream);
// recv[slot[t][j]] = gathered[r*T + t] for the j whose row lies on rank r
// (p.N = rank count, rows of rank r in [rank_offsets[r], rank_offsets[r+1]))
cudaError_t launch_rank_select(const RowMoveParams& p, const void* gathered, void* recv,
                               cudaStream_t stream);
// dst[t*k + j] = src[slot[t][j]]
cudaError_t launch_gather_rows(const RowMoveParams& p, const void* src, void* dst,
                               cudaStream_t stream);

// ---- combine -----------------------------------------------------------------
struct CombineParams {
    int64_t T;
    int k;
    size_t row_bytes;
    const int* slot;   // [T*k]; nullptr = rows t*k + j (contiguous source order)
    const float* w;    // [T*k]
    int* err;
    CopyEngine engine;
};
cudaError_t launch_combine(const CombineParams& p, const void* expert_out, void* y,
                           cudaStream_t stream);

// partial[r*T + t] = fp32 sum over the j whose row lies on rank r of
// w[t][j] * eo[slot[t][j]] (j order, FMA), for r < R
cudaError_t launch_combine_rank_partials(const CombineParams& p, int R, const int* rank_offsets,
                                         const void* expert_out, float* partial,
                                         cudaStream_t stream);
// y[t] = bf16_rne(sum over r in order of partial[r*T + t])
cudaError_t launch_reduce_rank_partials(const CombineParams& p, int R, const float* partial,
                                        void* y, cudaStream_t stream);

// ---- fp8 (e4m3) payload (fp8.cu) ------------------------------------------------
// hidden % 8 == 0, bf16 buffers 16-byte aligned, code buffers 8-byte aligned.
bool fp8_eligible(int64_t hidden, std::initializer_list<const void*> bf16_ptrs,
                  std::initializer_list<const void*> q_ptrs);
// Quantize `rows` bf16 rows (amax scale per row).  slot == nullptr: row r ->
// q row r; else row r goes to q rows dst_base[j] + slot[r*k + j] (j < k,
// slot >= 0; dst_base nullptr = 0), bounded by dst_rows.
cudaError_t launch_quantize_fp8(const void* src, int64_t rows, int64_t hidden, const int* slot, int k,
                                int64_t dst_rows, void* q, float* scale, int* err,
                                cudaStream_t stream, const int* dst_base = nullptr);
// Two-level fp8 dispatch in one kernel: each x row quantized once, its codes
// and scale stored to its staging row on every node touched, then each
// staging row read back and stored to the token's receive rows on that
// node.  Needs H % 16 == 0, H <= 8192, N + k <= 32 and 16-byte aligned x,
// staging and receive code buffers.
bool fp8_node_dispatch_eligible(const RowMoveParams& p, int64_t hidden,
                                std::initializer_list<const void*> ptrs);
cudaError_t launch_fp8_node_dispatch(const RowMoveParams& p, const void* x, int64_t hidden,
                                     void* staging_q, float* staging_scale, int64_t staging_rows,
                                     void* recv_q, float* recv_scale, cudaStream_t stream);
// y[t] = bf16_rne(sum_j fma(w[t][j] * scale[slot], decode(q[slot]), .))
cudaError_t launch_combine_fp8(const CombineParams& p, const void* q, const float* scale, void* y,
                               cudaStream_t stream);

// ---- expert parallelism over sharded sources (ep.cu) ----------------------------
// Receive buffers of at most kMaxEpRanks ranks, passed by value to kernels.
constexpr int kMaxEpRanks = 32;
struct EpParams {
    int64_t T;                        // this source's tokens
    int k, E, R, G, g;                // experts, expert ranks, sources, this source
    const int* topk;                  // [T*k] local routes
    const int* counts_all;            // [G*E] every source's expert counts
    const int* local_expert_offsets;  // [E+1] from the local layout
    const int* local_slot;            // [T*k] from the local layout
    int* expert_offsets;              // [E+1] out: rows of each expert, concatenated buffers
    int* rank_offsets;                // [R+1] out: first row of each rank's buffer
    int* slot;                        // [T*k] out: row of (t, j) in the concatenation
    int* err;
};
cudaError_t launch_ep_layout(const EpParams& p, cudaStream_t stream);
// bufs[r][slot[t][j] - rank_offsets[r]] = x[t] for the rank r holding the
// row (p.slot / p.rank_offsets are the sharded-source arrays, p.N = R);
// rows at or beyond capacity_rows of a buffer are refused (error bit).
cudaError_t launch_ep_dispatch(const RowMoveParams& p, const void* x, void* const* bufs,
                               int64_t capacity_rows, cudaStream_t stream);
// y[t] = bf16_rne(sum_j fma(w[t][j], bufs[r_j][slot[t][j] - rank_offsets[r_j]], .))
cudaError_t launch_ep_combine(const CombineParams& p, int R, const int* rank_offsets,
                              const void* const* bufs, int64_t capacity_rows, void* y,
                              cudaStream_t stream);

// ---- bulk-copy (TMA) engine (bulk.cu) ------------------------------------------
// Usable when the row size and every base address are multiples of 16 bytes.
bool bulk_eligible(size_t row_bytes, std::initializer_list<const void*> ptrs);
cudaError_t launch_dispatch_flat_bulk(const RowMoveParams& p, const void* x, void* recv,
                                      cudaStream_t stream);
cudaError_t launch_node_pack_bulk(const RowMoveParams& p, const void* x, void* staging,
                                  int64_t staging_rows, cudaStream_t stream);
cudaError_t launch_node_expand_bulk(const RowMoveParams& p, const void* staging,
                                    int64_t staging_rows, void* recv, cudaStream_t stream);
// Two-level dispatch in one kernel: per (token, chunk), the x chunk goes to
// the token's staging row of every node touched, and each staging row, once
// written, is read back and goes to the token's receive rows on its node.
// Needs N + k <= 32 (and 16-byte aligned rows, checked by the caller).
bool node_dispatch_eligible(const RowMoveParams& p);
cudaError_t launch_node_dispatch_bulk(const RowMoveParams& p, const void* x, void* staging,
                                      int64_t staging_rows, void* recv, cudaStream_t stream);
cudaError_t launch_combine_bulk(const CombineParams& p, const void* expert_out, void* y,
                                cudaStream_t stream);

}  // namespace moe

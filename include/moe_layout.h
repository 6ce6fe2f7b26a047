/*
 * moe_layout.h -- C ABI of the B200 MoE dispatch / combine library
 * (libmoe_layout.so).
 *
 * The library moves token rows between a batch of activations and an
 * expert-major receive buffer, the data shuffle of expert-parallel MoE, with
 * the layout transformation fused into the data movement.  Sources:
 *
 *  - FUSCO article (aigc.bar, "超DeepEP两倍！无问芯穹FUSCO如何以「空中变阵」
 *    突破MoE通信瓶颈"), section "传统 MoE 通信的痛点": decoupled designs pack
 *    scattered tokens into contiguous blocks before sending and unpack them
 *    after receiving; section "FUSCO 的核心创新": gather-send reads rows
 *    straight from their scattered locations by segment descriptor and
 *    scatter-recv writes them straight into the final layout; section
 *    "负载均衡与跨节点去重": one copy per destination node, fanned out
 *    inside the node by a forwarding GPU.
 *  - INC-MoE abstract: dispatch moves tokens to the holders of their
 *    selected experts, combine returns expert outputs to the token's owner.
 *  - TensorRT-LLM PR #13888 ("support non-divisible EP in MoE alltoall and
 *    slurm benchmark"): ceil/floor contiguous expert partitioning across
 *    ranks, a divisible fast path, and a clear error when num_experts <
 *    ep_size.
 *
 * Everything runs on one GPU.  Expert-parallel ranks and nodes are virtual:
 * rank r owns a contiguous range of receive rows, node n a contiguous range
 * of ranks.
 *
 * Conventions for every entry point
 *  - Pointers named "device" point to CUDA device memory of the current
 *    device; the caller allocates and owns all of it.  Nothing here
 *    allocates device memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Device work is enqueued on it asynchronously.
 *  - Argument and shape errors are detected on the host and returned before
 *    anything is enqueued.  Errors that depend on device data (an expert
 *    index out of range, a token naming one expert twice, a slot outside the
 *    receive buffer) are recorded in the layout's device error word and read
 *    back by moe_get_error(); kernels never trap.  When one is recorded the
 *    outputs of that call are unspecified, but every access stays inside the
 *    buffers described here.
 *  - A failed CUDA launch returns MOE_ERR_CUDA.
 *  - bf16 tensors are row-major [rows][hidden] 16-bit brain-float values.
 *    Rows whose byte size and base address are multiples of 16 take the
 *    vectorised kernels; other shapes are supported by narrower kernels.
 *  - The library keeps no state between calls other than per-device
 *    launch attributes; calls on different streams may run concurrently if
 *    their buffers do not overlap.
 */
#ifndef MOE_LAYOUT_H
#define MOE_LAYOUT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Size limits. */
#define MOE_MAX_EXPERTS 1024 /* experts per layer */
#define MOE_MAX_TOPK 32      /* experts per token */
#define MOE_MAX_NODES 32     /* virtual nodes when node staging is used */

/* moe_config_t.flags */
#define MOE_FLAG_TWO_LEVEL 0x1u  /* layout also builds node staging maps;
                                    dispatch goes through node staging */
#define MOE_FLAG_COPY_VECTOR 0x2u /* force the register (16-byte vector)
                                     copy kernels */
#define MOE_FLAG_COPY_BULK 0x4u   /* force the bulk-copy (TMA) kernels */
#define MOE_FLAG_LAYOUT_CLUSTER 0x8u /* layout in one thread-block-cluster
                                        launch (up to 131072 tokens) instead
                                        of the count/scan/assign kernels */
#define MOE_FLAG_LAYOUT_FUSED 0x10u  /* moe_layout_dispatch(): a count kernel
                                        and an assign/dispatch kernel instead
                                        of the layout kernels and the
                                        dispatch kernel (flat layouts) */
#define MOE_FLAG_TWO_LEVEL_FUSED 0x20u /* two-level dispatch in one kernel
                                          that reads each staging row back
                                          right after writing it (the
                                          default where it applies; the flag
                                          is accepted and changes nothing) */
#define MOE_FLAG_TWO_LEVEL_SPLIT 0x40u /* two-level dispatch as a pack kernel
                                          then an expansion kernel */

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* null pointer, size out of range, bad flag */
    MOE_ERR_EMPTY_RANK = 2,  /* num_experts < num_ranks: some rank would
                                hold no expert (PR #13888 review thread) */
    MOE_ERR_BAD_NODES = 3,   /* num_nodes does not divide num_ranks, or too
                                many nodes for node staging */
    MOE_ERR_EXPERT_OOB = 4,  /* device data: expert index outside [0, E) */
    MOE_ERR_DUP_EXPERT = 5,  /* device data: a token names an expert twice */
    MOE_ERR_TIMEOUT = 6,     /* device: a bounded wait gave up */
    MOE_ERR_CUDA = 7,        /* a CUDA call failed */
    MOE_ERR_BAD_LAYOUT = 8   /* device data: a slot outside the receive
                                buffer was met by dispatch or combine */
} moe_status_t;

/* Shape of one dispatch/combine problem.
 *   num_tokens  T >= 0 tokens in the batch (T * top_k < 2^31)
 *   hidden      H >= 1 bf16 values per token row
 *   num_experts E, 1 <= E <= MOE_MAX_EXPERTS
 *   top_k       k experts per token, 1 <= k <= min(E, MOE_MAX_TOPK)
 *   num_ranks   R virtual expert-parallel ranks, 1 <= R <= E
 *   num_nodes   N virtual nodes, N divides R (R/N ranks per node)
 *   flags       MOE_FLAG_* bits */
typedef struct moe_config {
    int64_t num_tokens;
    int32_t hidden;
    int32_t num_experts;
    int32_t top_k;
    int32_t num_ranks;
    int32_t num_nodes;
    uint32_t flags;
} moe_config_t;

/* Layout metadata ("segment descriptors"), all device int32 arrays owned by
 * the caller.  The receive buffer has exactly T*k rows, expert-major: the
 * rows of expert e are [expert_offsets[e], expert_offsets[e+1]) in
 * ascending token order; rank r owns rows [rank_offsets[r],
 * rank_offsets[r+1]).
 *   expert_counts  [E]     rows per expert
 *   expert_offsets [E+1]   exclusive prefix of expert_counts
 *   rank_offsets   [R+1]   first row of each rank (last = T*k)
 *   slot           [T*k]   receive row of (token t, column j), row-major
 *   node_counts    [N]     tokens touching node n          (TWO_LEVEL)
 *   node_offsets   [N+1]   exclusive prefix of node_counts (TWO_LEVEL)
 *   node_slot      [T*N]   rank of token t among the tokens touching node n,
 *                          or -1 when t touches no expert of n (TWO_LEVEL)
 *   error_word     [1]     device error bits; zero it once before first use,
 *                          moe_get_error() reads and clears it
 *   workspace      moe_layout_workspace_bytes() bytes, 16-byte aligned.
 *                          Scratch for moe_layout; without
 *                          MOE_FLAG_TWO_LEVEL it also holds a counter used by
 *                          moe_layout_dispatch with MOE_FLAG_LAYOUT_FUSED, so
 *                          zero the whole workspace once before its first
 *                          use (every call leaves the counter zero; calls
 *                          that share a workspace must not overlap on the
 *                          GPU)
 *   node_src       [moe_node_staging_rows()]  token held by each staging row:
 *                          node_src[node_offsets[n] + node_slot[t][n]] = t
 *                          (TWO_LEVEL, optional).  When it is given,
 *                          moe_layout writes it and the second phase of a
 *                          two-level dispatch divides its work by staging
 *                          rows, so a node that receives many more tokens
 *                          than the others is spread over the whole GPU
 *                          (the load-aware forwarding of the FUSCO article,
 *                          section "FUSCO 的核心创新"); when it is NULL the
 *                          second phase walks (node, token) pairs, whose
 *                          work per node follows that node's load.  Only
 *                          entries below node_offsets[N] are written.
 * Node arrays may be NULL when MOE_FLAG_TWO_LEVEL is not set. */
typedef struct moe_layout {
    int32_t *expert_counts;
    int32_t *expert_offsets;
    int32_t *rank_offsets;
    int32_t *slot;
    int32_t *node_counts;
    int32_t *node_offsets;
    int32_t *node_slot;
    int32_t *error_word;
    void *workspace;
    int32_t *node_src;
} moe_layout_t;

/* Text of a status code (static storage, never NULL). */
const char *moe_status_string(moe_status_t status);

/* Host-side check of a configuration (the same check every entry point
 * runs first).  Order of checks: basic ranges (MOE_ERR_INVALID_ARG), then
 * E < R (MOE_ERR_EMPTY_RANK), then the node grouping (MOE_ERR_BAD_NODES). */
moe_status_t moe_check_config(const moe_config_t *cfg);

/* Ceil/floor contiguous expert partition (PR #13888, PR description and
 * the divisible-fast-path commit): base = E / R, rem = E % R; ranks 0 ..
 * rem-1 hold base+1 consecutive experts, the others base.  Writes
 * rank_first_expert[0..R] (host array, R+1 entries, last = E).  Host only.
 * Errors: MOE_ERR_INVALID_ARG for E < 1, R < 1 or a NULL array;
 * MOE_ERR_EMPTY_RANK for E < R. */
moe_status_t moe_expert_partition(int32_t num_experts, int32_t num_ranks,
                                  int32_t *rank_first_expert);

/* Bytes of moe_layout_t.workspace needed by moe_layout() for cfg. */
moe_status_t moe_layout_workspace_bytes(const moe_config_t *cfg, size_t *bytes);

/* Rows a node staging buffer must hold for cfg: T * min(N, k). */
moe_status_t moe_node_staging_rows(const moe_config_t *cfg, int64_t *rows);

/* Layout: per-expert histograms of 256-token chunks, an exclusive scan over
 * experts and chunks (expert e's first row in chunk c is expert_offsets[e]
 * plus e's rows in chunks before c), and stable slot assignment (FUSCO
 * article, "FUSCO 的核心创新": the segment descriptors that drive
 * gather-send / scatter-recv).
 *   topk_idx  device int32 [T*k], row-major [T][k], the router's choices
 *   layout    device arrays as described above (TWO_LEVEL: node arrays too)
 * Data errors go to layout->error_word. */
moe_status_t moe_layout(const moe_config_t *cfg, const int32_t *topk_idx,
                        const moe_layout_t *layout, void *stream);

/* Fused dispatch (gather-send / scatter-recv): recv[slot[t][j]] = x[t] for
 * every (t, j); each x row is read once and written straight to all its
 * destination rows, with no pack or unpack pass.
 *   x             device bf16 [T][H]
 *   recv          device bf16 [T*k][H]
 *   node_staging  device bf16 [moe_node_staging_rows()][H] when
 *                 MOE_FLAG_TWO_LEVEL is set (NULL otherwise): rows are first
 *                 written once per (token, node touched), node-major then
 *                 token order (FUSCO article, "负载均衡与跨节点去重"), then
 *                 expanded from staging to the expert rows of that node.
 *                 The final recv is identical in both modes.
 * Two-level engines: with 16-byte aligned rows and N + k <= 32, one kernel
 * does both phases, reading each staging row back right after writing it
 * (the reads then come from L2, so the staging rows cross HBM once).  With
 * MOE_FLAG_TWO_LEVEL_SPLIT or MOE_FLAG_COPY_VECTOR, or where the one kernel
 * does not apply, a pack kernel writes the staging rows and an expansion
 * kernel reads them back.  Measured on B200 on the DeepSeek-V3-shaped
 * workload in the same build, the one-kernel form's step (layout, dispatch,
 * combine) took 764 us against 808 us for the two kernels; with later
 * kernels the one-kernel step is about 719 us. */
moe_status_t moe_dispatch(const moe_config_t *cfg, const moe_layout_t *layout,
                          const void *x, void *recv, void *node_staging,
                          void *stream);

/* Layout and dispatch in one call, the layout transformation fused with
 * the data movement (FUSCO article, "FUSCO 的核心创新": the transfer itself
 * carries where each row comes from and goes to).  Same results as
 * moe_layout() followed by moe_dispatch() with the same arguments.
 *  - By default the layout kernels run first and the dispatch kernel starts
 *    loading x rows while they still run (bulk-copy engine), because x and
 *    topk_idx are complete when the layout starts.
 *  - With MOE_FLAG_LAYOUT_FUSED, without MOE_FLAG_TWO_LEVEL, with 16-byte
 *    aligned x, recv and workspace, H*2 a multiple of 16 and E <= 256, it is
 *    two kernels over the same split of the tokens (one CTA per SM): a count
 *    kernel whose last CTA turns the per-CTA histograms into prefixes and
 *    offsets, and an assign/dispatch kernel that loads its x rows and routes
 *    while the count kernel runs, then ranks its tokens and stores each row
 *    straight to its receive rows.  A ticket counter lives in the workspace
 *    (zero it once before first use).  Other configurations with this flag
 *    take the default path.
 * Arguments as for moe_layout() and moe_dispatch(); all are checked before
 * anything is enqueued. */
moe_status_t moe_layout_dispatch(const moe_config_t *cfg, const int32_t *topk_idx,
                                 const moe_layout_t *layout, const void *x, void *recv,
                                 void *node_staging, void *stream);

/* Fused combine: y[t] = bf16_rne( sum_{j=0..k-1} w[t][j] * eo[slot[t][j]] ),
 * accumulated in fp32 with one fused multiply-add per j in column order,
 * starting from +0 (INC-MoE abstract: combine returns expert outputs to the
 * token's owner; the order and precision are this library's choice).
 *   expert_out    device bf16 [T*k][H], receive-buffer layout
 *   topk_weights  device fp32 [T][k], used as given
 *   y             device bf16 [T][H]
 * Large combines (at least 8 resident waves of (token, 1 KB row chunk) work
 * items) whose rows are a multiple of 32 bytes, with expert_out and y 32-byte
 * aligned, move 32 bytes per lane per access (sm_100's 256-bit loads and
 * stores); the results are the same bit for bit either way. */
moe_status_t moe_combine(const moe_config_t *cfg, const moe_layout_t *layout,
                         const void *expert_out, const float *topk_weights,
                         void *y, void *stream);

/* Waits for `stream`, reads and clears layout->error_word, and returns the
 * recorded error: MOE_ERR_EXPERT_OOB before MOE_ERR_DUP_EXPERT before
 * MOE_ERR_BAD_LAYOUT before MOE_ERR_TIMEOUT; MOE_OK when none. */
moe_status_t moe_get_error(const moe_layout_t *layout, void *stream);

/* ---- decoupled comparison path (pack -> contiguous copy -> unpack) ----
 * The design the FUSCO article ("传统 MoE 通信的痛点") measures reorder
 * passes against: rows are first packed into contiguous per-destination
 * blocks, the blocks are moved by one contiguous copy, and the receiver
 * unpacks them into the final layout.  Results equal moe_dispatch /
 * moe_combine bit for bit. */

/* Dispatch, decoupled.  `cfg` must have num_nodes == num_ranks (<=
 * MOE_MAX_NODES) and MOE_FLAG_TWO_LEVEL, and `layout` must come from
 * moe_layout() with that cfg, so its node arrays are per-rank blocks.
 * Pack: x[t] -> send, once per (token, rank touched), rank-major then token
 * order.  Copy: send -> xfer (node_offsets[R] rows, read on the device).
 * Unpack: each xfer row -> the token's expert rows on that rank.
 *   send, xfer  device bf16 [moe_node_staging_rows(cfg)][H] each. */
moe_status_t moe_dispatch_decoupled(const moe_config_t *cfg,
                                    const moe_layout_t *layout, const void *x,
                                    void *send, void *xfer, void *recv,
                                    void *stream);

/* Combine, decoupled.  Pack: send[t*k + j] = expert_out[slot[t][j]] (source
 * order).  Copy: send -> xfer (T*k rows).  Unpack: y[t] = the same fp32 sum
 * as moe_combine, read from the contiguous rows xfer[t*k .. t*k+k-1].
 *   send, xfer  device bf16 [T*k][H] each. */
moe_status_t moe_combine_decoupled(const moe_config_t *cfg,
                                   const moe_layout_t *layout,
                                   const void *expert_out,
                                   const float *topk_weights, void *send,
                                   void *xfer, void *y, void *stream);

/* ---- AllGather / ReduceScatter comparison path ----
 * The collective formulation of dispatch and combine: INC-MoE abstract
 * (dispatch as an in-network AllGather, combine as a ReduceScatter) and the
 * AllGather + ReduceScatter fallback of TensorRT-LLM PR #13888.  On one GPU
 * the R virtual ranks are regions of HBM.  Requires num_ranks <=
 * MOE_MAX_NODES and a layout from moe_layout() with the same cfg. */

/* Dispatch, all-gather form.  All-gather: every rank r receives a copy of
 * every token, gathered[r*T + t] = x[t].  Select: rank r copies, from its
 * gathered rows, each token's rows on its experts into recv (rank r's rows
 * are [rank_offsets[r], rank_offsets[r+1])).  recv equals moe_dispatch()'s
 * bit for bit.
 *   gathered  device bf16 [R*T][H] */
moe_status_t moe_dispatch_allgather(const moe_config_t *cfg, const moe_layout_t *layout,
                                    const void *x, void *gathered, void *recv, void *stream);

/* Combine, reduce-scatter form.  Every rank r sums, for every token, the
 * weighted rows of its own experts in fp32 (one FMA per column j in order,
 * from +0) into partial[r*T + t]; then y[t] = bf16_rne(partial[0*T+t] +
 * partial[1*T+t] + ... ) added in rank order from +0.  Agrees with
 * moe_combine() within the combine tolerance (the additions are ordered
 * differently).
 *   partial  device fp32 [R*T][H] */
moe_status_t moe_combine_reducescatter(const moe_config_t *cfg, const moe_layout_t *layout,
                                       const void *expert_out, const float *topk_weights,
                                       float *partial, void *y, void *stream);

/* ---- expert parallelism over sharded sources ----
 * With one rank per GPU, rank g routes only its own T_g tokens and every
 * rank's receive buffer holds its own experts' rows ("[None][feat] support
 * non-divisible EP in MoE alltoall and slurm benchmark", TensorRT-LLM PR
 * #13888: the NVLinkOneSided dispatch writes straight into peer receive
 * buffers; FUSCO article, "FUSCO 的核心创新": every row goes straight to its
 * final position).  Order inside rank r's buffer: expert-major, then source
 * rank, then the source's token order.  When the sources are contiguous token
 * ranges of one batch in rank order, the rows equal moe_layout()'s on the
 * whole batch.  One step on rank g:
 *   1. moe_layout(cfg_g, topk_g, local) over its own tokens (cfg_g.num_tokens
 *      = T_g, flat, num_ranks = R): local->expert_counts are its counts;
 *   2. the caller gathers every rank's expert_counts into counts_all
 *      ([G][E], device, source-major), e.g. with an NCCL all-gather;
 *   3. moe_ep_layout(): the rows of the concatenated receive buffers;
 *   4. moe_ep_dispatch() into the R receive buffers (peer-mapped pointers),
 *      then a barrier across ranks, the experts, another barrier, and
 *   5. moe_ep_combine() from the R expert-output buffers.
 * No entry point synchronises ranks; barriers and buffer mapping are the
 * caller's.  num_ranks <= MOE_MAX_NODES, and MOE_FLAG_TWO_LEVEL is refused. */

/* Rows in the concatenation of all ranks' receive buffers (device int32,
 * caller-owned):
 *   expert_offsets [E+1]   first row of each expert (last = total rows)
 *   rank_offsets   [R+1]   rank r's buffer holds rows [rank_offsets[r],
 *                          rank_offsets[r+1]); its local row is the
 *                          difference from rank_offsets[r]
 *   slot           [T_g*k] row of this rank's (t, j), -1 if the route was
 *                          invalid */
typedef struct moe_ep_layout {
    int32_t *expert_offsets;
    int32_t *rank_offsets;
    int32_t *slot;
} moe_ep_layout_t;

/* Rows every expert rank receives, from the gathered counts of step 2 (host
 * arithmetic only, for sizing the receive and expert-output buffers before
 * the first step): rows_out[r] = the sum over sources g and over rank r's
 * experts e (the ceil/floor contiguous partition of moe_expert_partition())
 * of counts_all[g][e].  These equal the differences of the rank_offsets
 * that moe_ep_layout() writes.
 *   counts_all  HOST int32 [num_sources][num_experts], every count >= 0
 *   rows_out    HOST int64 [num_ranks]
 * Errors (nothing written): MOE_ERR_INVALID_ARG for a NULL pointer, a size
 * below 1 or a negative count; MOE_ERR_EMPTY_RANK when num_experts <
 * num_ranks. */
moe_status_t moe_ep_receive_rows(int32_t num_experts, int32_t num_ranks, int32_t num_sources,
                                 const int32_t *counts_all, int64_t *rows_out);

/* Let kernels that run on `device` load from and store to memory that
 * lives on `peer_device`: another rank's receive and expert-output buffers,
 * mapped into this process (e.g. CUDA IPC handles opened by the caller).
 * Host call; nothing is enqueued, and the calling thread's current device is
 * restored.  Enabling a pair that is already enabled is not an error.
 * Errors: MOE_ERR_INVALID_ARG for a device index out of range or device ==
 * peer_device; MOE_ERR_CUDA when the two devices cannot reach each other
 * (or no device is present). */
moe_status_t moe_enable_peer_access(int32_t device, int32_t peer_device);

/* Step 3.  cfg: this rank's shard (as in step 1); source_rank g in
 * [0, num_sources); counts_all: device int32 [num_sources][E] with row g equal
 * to local->expert_counts; topk_idx: the shard's routes; local: the layout of
 * step 1 (its expert_offsets, slot and error_word are read).  Every rank
 * computes the same expert_offsets and rank_offsets. */
moe_status_t moe_ep_layout(const moe_config_t *cfg, int32_t source_rank, int32_t num_sources,
                           const int32_t *topk_idx, const int32_t *counts_all,
                           const moe_layout_t *local, const moe_ep_layout_t *ep, void *stream);

/* Step 4: bufs[r][slot[t][j] - rank_offsets[r]] = x[t] for every (t, j).
 *   recv_bufs     HOST array of num_ranks device pointers (this GPU's or
 *                 peers', e.g. CUDA IPC mappings), each bf16 rows of `hidden`
 *   capacity_rows rows each buffer holds; a row at or beyond it is skipped
 *                 and reported (MOE_ERR_BAD_LAYOUT) */
moe_status_t moe_ep_dispatch(const moe_config_t *cfg, const moe_layout_t *local,
                             const moe_ep_layout_t *ep, const void *x, void *const *recv_bufs,
                             int64_t capacity_rows, void *stream);

/* Step 5: y[t] = bf16_rne( sum_{j=0..k-1} w[t][j] * eo_r[slot[t][j] -
 * rank_offsets[r]] ), r the rank holding the row, fp32 FMA in column order
 * as in moe_combine().
 *   expert_out_bufs  HOST array of num_ranks device pointers, bf16 rows laid
 *                    out like the receive buffers */
moe_status_t moe_ep_combine(const moe_config_t *cfg, const moe_layout_t *local,
                            const moe_ep_layout_t *ep, const void *const *expert_out_bufs,
                            int64_t capacity_rows, const float *topk_weights, void *y,
                            void *stream);

/* ---- fp8 (e4m3) payload ----
 * TensorRT-LLM PR #13888 (ConfigurableMoE commit) validates an fp8
 * low-precision combine at rtol 0.02 / atol 0.15.  Rows are carried as OCP
 * E4M3 codes (1 byte per value) with one fp32 scale per row: scale = amax /
 * 448 (a zero row uses 1) and code = e4m3(v * (448 / amax)), round to
 * nearest even, saturated to +-448.  Requirements: hidden % 8 == 0, bf16
 * buffers 16-byte aligned, code buffers 8-byte aligned (else
 * MOE_ERR_INVALID_ARG). */

/* Quantize `rows` bf16 rows of `hidden` values (e.g. expert outputs).
 *   src    device bf16 [rows][hidden]
 *   q      device uint8 [rows][hidden] e4m3 codes
 *   scale  device fp32 [rows] */
moe_status_t moe_quantize_rows_fp8(const void *src, int64_t rows, int32_t hidden, void *q,
                                   float *scale, void *stream);

/* Fused dispatch with an fp8 payload: each x row is quantized once and its
 * codes and scale are written to all its receive rows (flat mode only;
 * MOE_FLAG_TWO_LEVEL gives MOE_ERR_INVALID_ARG).
 *   recv_q      device uint8 [T*k][H]
 *   recv_scale  device fp32 [T*k] */
moe_status_t moe_dispatch_fp8(const moe_config_t *cfg, const moe_layout_t *layout, const void *x,
                              void *recv_q, float *recv_scale, void *stream);

/* Two-level dispatch with an fp8 payload (MOE_FLAG_TWO_LEVEL required):
 * each x row is quantized once, into the staging row of every node it
 * touches (codes and scale, as moe_dispatch() stages bf16 rows), and the
 * node expansion then copies codes and scales to the receive rows.  With
 * H % 16 == 0, H <= 8192, N + k <= 32 and 16-byte aligned x and code
 * buffers one kernel does both phases (each staging row read back from L2
 * right after it is written); MOE_FLAG_TWO_LEVEL_SPLIT or other shapes take
 * a quantizer and two expansion kernels.  Results equal moe_dispatch_fp8()
 * on the same layout bit for bit.
 *   staging_q      device uint8 [moe_node_staging_rows()][H]
 *   staging_scale  device fp32 [moe_node_staging_rows()]
 *   recv_q, recv_scale  as for moe_dispatch_fp8() */
moe_status_t moe_dispatch_fp8_two_level(const moe_config_t *cfg, const moe_layout_t *layout,
                                        const void *x, void *staging_q, float *staging_scale,
                                        void *recv_q, float *recv_scale, void *stream);

/* Fused combine of fp8 expert rows: coef_j = w[t][j] * scale[slot[t][j]]
 * (fp32), acc = fma(coef_j, decode(code), acc) for j = 0..k-1 from +0, one
 * bf16 round-to-nearest-even store.
 *   eo_q      device uint8 [T*k][H] (receive-buffer layout)
 *   eo_scale  device fp32 [T*k] */
moe_status_t moe_combine_fp8(const moe_config_t *cfg, const moe_layout_t *layout,
                             const void *eo_q, const float *eo_scale, const float *topk_weights,
                             void *y, void *stream);

/* ---- layout without caller-provided scratch ----
 * No counterpart on the pages: this entry point exists for callers that
 * cannot allocate device memory (for example code that runs while a stream
 * is being captured and may not allocate, runtimes without a device
 * allocator, or plugins whose host framework owns every allocation).
 *
 * Same inputs, outputs and results as moe_layout(), but the layout's
 * scratch comes from a fixed array of MOE_LAYOUT_NOALLOC_SCRATCH_BYTES bytes
 * inside the library's device memory (held on every GPU that loads the
 * library until the process exits); layout->workspace is ignored and may be
 * NULL.  Nothing is allocated.
 *  - Limit: the layout's scratch is its per-chunk histograms, 4 * E *
 *    ceil(T / 256) bytes, plus 4 * N * ceil(T / 256) with MOE_FLAG_TWO_LEVEL,
 *    each rounded up to 256 bytes.  Configurations that need more than
 *    MOE_LAYOUT_NOALLOC_SCRATCH_BYTES are refused with MOE_ERR_INVALID_ARG
 *    before anything is enqueued (e.g. E = 256 allows T up to 1,048,576).
 *  - Every call looks up the array's device address on the current device
 *    (a host-side lookup, nothing is enqueued).  The first call on a device
 *    may also load the library's device code there; make that first call
 *    before any stream capture.
 *  - All calls on a device share the one array: calls that overlap on the
 *    GPU (other streams, or other threads' streams) race and give wrong
 *    layouts.  Order them on one stream or with events.
 *  - The array keeps the last call's contents; a call reads only what it
 *    wrote itself, so nothing needs clearing between calls. */
#define MOE_LAYOUT_NOALLOC_SCRATCH_BYTES (4u << 20)
moe_status_t moe_layout_noalloc(const moe_config_t *cfg, const int32_t *topk_idx,
                                const moe_layout_t *layout, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_LAYOUT_H */

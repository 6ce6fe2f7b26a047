/*
 * moe_oracle.c -- plain, slow, obviously-correct CPU oracle for MoE
 * expert-parallel dispatch and combine with their layout metadata.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file.  Only the test suite, the package smoke check and the
 * CPU-baseline leg of the benchmark use it.  It shares no code, header,
 * table or helper with the CUDA library; the two meet only through the
 * seeded input generator.
 *
 * What it computes, and where the pages say so:
 *
 *  - Expert -> rank partition.  "[None][feat] support non-divisible EP in MoE
 *    alltoall and slurm benchmark" (TensorRT-LLM PR #13888), PR description
 *    ("ceil/floor contiguous partitioning") and the commit that adds the
 *    divisible fast path (base = E / R, remainder = E mod R, example 256
 *    experts on 7 ranks -> base 36, remainder 4).  Reading taken: ranks are
 *    filled in order with contiguous experts and the first `remainder` ranks
 *    hold one extra expert.  Here that is a plain loop over ranks, not the
 *    closed form.
 *  - E < R is refused up front.  Same PR, review thread on num_experts <
 *    ep_size (a clear error instead of ranks with no experts).
 *  - Layout ("segment descriptors").  FUSCO article (aigc.bar), section
 *    "FUSCO 的核心创新": gather-send reads scattered rows by segment
 *    descriptor, scatter-recv writes each row straight into its final
 *    position.  The descriptor contents are not given; the reading taken is
 *    an expert-major receive buffer of exactly T*k rows, ordered inside each
 *    expert by ascending token index, with per-expert counts/offsets,
 *    per-rank offsets and a per-(token, slot) destination row.
 *  - Dispatch.  INC-MoE abstract (dispatch moves each token to the devices
 *    hosting its selected experts) and the FUSCO article section above: one
 *    copy of x[t] lands in every destination row of token t.
 *  - Two-level dispatch.  FUSCO article, section "负载均衡与跨节点去重":
 *    a token bound for several GPUs of one node crosses nodes once, to a
 *    forwarding GPU that fans it out inside the node.  Here: one staging row
 *    per (token, node touched), node-major then token order, then expansion
 *    from staging to the expert rows of that node.
 *  - Combine.  INC-MoE abstract (combine returns expert outputs to each
 *    token's owner) with the reduction by gate weight.  The pages fix no
 *    order or precision; the reading taken is fp32 accumulation with one
 *    fused multiply-add per selected expert in top-k column order j = 0..k-1,
 *    starting from +0.0f, and one round-to-nearest-even store to bf16.
 *
 * Build: cc -std=c99 -O2 -ffp-contract=off -shared -fPIC (so that the only
 * fused multiply-add is the explicit fmaf call).
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <math.h>

/* Status codes.  Their meaning mirrors the library's public status enum by
 * convention (same numbers, same meaning); they are defined here on their
 * own so the oracle needs no header of the library. */
enum {
    ORC_OK = 0,
    ORC_INVALID_ARG = 1,
    ORC_EMPTY_RANK = 2,
    ORC_BAD_NODES = 3,
    ORC_EXPERT_OOB = 4,
    ORC_DUP_EXPERT = 5
};

/* ------------------------------------------------------------------ */
/* bf16 <-> fp32, from the IEEE-754 binary32 layout                    */
/* ------------------------------------------------------------------ */

/* bf16 is the upper half of a binary32: widening is a 16-bit shift. */
float oracle_bf16_to_f32(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Narrowing with round-to-nearest, ties-to-even, written from the
 * definition: keep the upper 16 bits, look at the 16 discarded bits, round
 * up when they exceed one half, or equal one half and the kept part is odd.
 * A carry out of the mantissa moves into the exponent, which is the correct
 * result (up to and including overflow to infinity).  NaN stays NaN: the
 * sign and upper payload are kept and the quiet bit is forced so that the
 * truncated payload can never read as infinity. */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint32_t exp_bits = (u >> 23) & 0xFFu;
    uint32_t man_bits = u & 0x7FFFFFu;
    if (exp_bits == 0xFFu && man_bits != 0u)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t kept = u >> 16;
    uint32_t dropped = u & 0xFFFFu;
    int round_up = 0;
    if (dropped > 0x8000u)
        round_up = 1;
    else if (dropped == 0x8000u && (kept & 1u))
        round_up = 1;
    return (uint16_t)(kept + (uint32_t)round_up);
}

void oracle_f32_to_bf16_array(const float *src, uint16_t *dst, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = oracle_f32_to_bf16(src[i]);
}

void oracle_bf16_to_f32_array(const uint16_t *src, float *dst, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = oracle_bf16_to_f32(src[i]);
}

/* ------------------------------------------------------------------ */
/* Partition                                                           */
/* ------------------------------------------------------------------ */

/* Fill rank_first_expert[0..R] by walking the ranks in order and giving each
 * one base experts, plus one more while the remainder lasts. */
int oracle_partition(int32_t E, int32_t R, int32_t *rank_first_expert)
{
    if (E < 1 || R < 1 || rank_first_expert == NULL)
        return ORC_INVALID_ARG;
    if (E < R)
        return ORC_EMPTY_RANK;
    int32_t base = E / R;
    int32_t extra_left = E - base * R;
    int32_t next = 0;
    for (int32_t r = 0; r < R; ++r) {
        rank_first_expert[r] = next;
        int32_t size = base;
        if (extra_left > 0) {
            size += 1;
            extra_left -= 1;
        }
        next += size;
    }
    rank_first_expert[R] = next;
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Validation                                                          */
/* ------------------------------------------------------------------ */

int oracle_validate_config(int64_t T, int32_t H, int32_t E, int32_t k,
                           int32_t R, int32_t N)
{
    if (T < 0 || H < 1 || E < 1 || R < 1 || N < 1 || k < 1)
        return ORC_INVALID_ARG;
    if (k > E)
        return ORC_INVALID_ARG;
    if (E < R)
        return ORC_EMPTY_RANK;
    if (N > R || (R % N) != 0)
        return ORC_BAD_NODES;
    return ORC_OK;
}

/* Every index lies in [0, E) and no token names one expert twice.  An
 * out-of-range index is reported before a repeat when both occur. */
int oracle_validate_topk(int64_t T, int32_t k, int32_t E, const int32_t *topk)
{
    int any_dup = 0;
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t j = 0; j < k; ++j) {
            int32_t e = topk[t * k + j];
            if (e < 0 || e >= E)
                return ORC_EXPERT_OOB;
            for (int32_t i = 0; i < j; ++i)
                if (topk[t * k + i] == e)
                    any_dup = 1;
        }
    }
    return any_dup ? ORC_DUP_EXPERT : ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Layout                                                              */
/* ------------------------------------------------------------------ */

/* topk:            int32 [T][k] row-major
 * expert_counts:   int32 [E]
 * expert_offsets:  int32 [E+1]   exclusive prefix of counts
 * rank_offsets:    int32 [R+1]   first receive row of each rank
 * slot:            int32 [T][k]  destination row of (t, j)
 * node_counts:     int32 [N]     tokens touching node n   (optional)
 * node_offsets:    int32 [N+1]   exclusive prefix         (optional)
 * node_slot:       int32 [T][N]  rank of t among tokens touching n, or -1
 *                                                         (optional)
 * The three node arrays are either all NULL or all given. */
int oracle_layout(int64_t T, int32_t k, int32_t E, int32_t R, int32_t N,
                  const int32_t *topk,
                  int32_t *expert_counts, int32_t *expert_offsets,
                  int32_t *rank_offsets, int32_t *slot,
                  int32_t *node_counts, int32_t *node_offsets,
                  int32_t *node_slot)
{
    int st = oracle_validate_config(T, 1, E, k, R, N);
    if (st != ORC_OK)
        return st;
    st = oracle_validate_topk(T, k, E, topk);
    if (st != ORC_OK)
        return st;

    /* counts, then offsets as an exclusive prefix sum over experts */
    for (int32_t e = 0; e < E; ++e)
        expert_counts[e] = 0;
    for (int64_t t = 0; t < T; ++t)
        for (int32_t j = 0; j < k; ++j)
            expert_counts[topk[t * k + j]] += 1;
    int64_t run = 0;
    for (int32_t e = 0; e < E; ++e) {
        expert_offsets[e] = (int32_t)run;
        run += expert_counts[e];
    }
    expert_offsets[E] = (int32_t)run;

    int32_t *first = (int32_t *)malloc(sizeof(int32_t) * (size_t)(R + 1));
    if (first == NULL)
        return ORC_INVALID_ARG;
    oracle_partition(E, R, first);
    for (int32_t r = 0; r <= R; ++r)
        rank_offsets[r] = expert_offsets[first[r]];

    /* slots: one cursor per expert, walked in token order */
    int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    if (cursor == NULL) {
        free(first);
        return ORC_INVALID_ARG;
    }
    for (int32_t e = 0; e < E; ++e)
        cursor[e] = expert_offsets[e];
    for (int64_t t = 0; t < T; ++t)
        for (int32_t j = 0; j < k; ++j) {
            int32_t e = topk[t * k + j];
            slot[t * k + j] = cursor[e];
            cursor[e] += 1;
        }
    free(cursor);

    if (node_counts != NULL && node_offsets != NULL && node_slot != NULL) {
        int32_t ranks_per_node = R / N;
        int32_t *node_of_expert = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
        int32_t *ncursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
        if (node_of_expert == NULL || ncursor == NULL) {
            free(node_of_expert);
            free(ncursor);
            free(first);
            return ORC_INVALID_ARG;
        }
        for (int32_t r = 0; r < R; ++r)
            for (int32_t e = first[r]; e < first[r + 1]; ++e)
                node_of_expert[e] = r / ranks_per_node;
        for (int32_t n = 0; n < N; ++n)
            ncursor[n] = 0;
        for (int64_t t = 0; t < T; ++t) {
            for (int32_t n = 0; n < N; ++n) {
                int touched = 0;
                for (int32_t j = 0; j < k; ++j)
                    if (node_of_expert[topk[t * k + j]] == n)
                        touched = 1;
                if (touched) {
                    node_slot[t * N + n] = ncursor[n];
                    ncursor[n] += 1;
                } else {
                    node_slot[t * N + n] = -1;
                }
            }
        }
        int64_t nrun = 0;
        for (int32_t n = 0; n < N; ++n) {
            node_counts[n] = ncursor[n];
            node_offsets[n] = (int32_t)nrun;
            nrun += ncursor[n];
        }
        node_offsets[N] = (int32_t)nrun;
        free(node_of_expert);
        free(ncursor);
    }
    free(first);
    return ORC_OK;
}

/* Layout with the source tokens sharded over G ranks (expert parallelism
 * over real GPUs; "[None][feat] support non-divisible EP in MoE alltoall and
 * slurm benchmark", TensorRT-LLM PR #13888, the NVLinkOneSided one-sided
 * dispatch of the commit adding the divisible fast path, and the FUSCO
 * article, section "FUSCO 的核心创新", rows written straight to their final
 * position).  Source rank g holds tokens [shard_begin[g], shard_begin[g+1]).
 * The pages give no receive order across sources; the reading taken is
 * expert-major, then source rank, then the source's token order, each
 * receiving rank's rows contiguous.  Steps, as a sharded system takes them:
 *  1. every source counts its own routes per expert: counts[g][e];
 *  2. the counts are exchanged, so every rank sees counts[*][e];
 *  3. expert totals, their exclusive prefix (expert_offsets) and the rank
 *     offsets of the ceil/floor partition;
 *  4. the first row of source g inside expert e: expert_offsets[e] plus the
 *     counts of the sources before g;
 *  5. each source walks its tokens in order with one cursor per expert.
 * slot[t][j] is the row in the concatenation of all ranks' receive buffers
 * (rank r holds rows [rank_offsets[r], rank_offsets[r+1])). */
int oracle_ep_layout(int64_t T, int32_t k, int32_t E, int32_t R, int32_t G,
                     const int64_t *shard_begin, const int32_t *topk,
                     int32_t *counts, int32_t *expert_offsets,
                     int32_t *rank_offsets, int32_t *slot)
{
    int st = oracle_validate_config(T, 1, E, k, R, 1);
    if (st != ORC_OK)
        return st;
    st = oracle_validate_topk(T, k, E, topk);
    if (st != ORC_OK)
        return st;
    if (G < 1 || shard_begin[0] != 0 || shard_begin[G] != T)
        return ORC_INVALID_ARG;
    for (int32_t g = 0; g < G; ++g)
        if (shard_begin[g + 1] < shard_begin[g])
            return ORC_INVALID_ARG;

    /* 1. per-source histograms */
    for (int64_t i = 0; i < (int64_t)G * E; ++i)
        counts[i] = 0;
    for (int32_t g = 0; g < G; ++g)
        for (int64_t t = shard_begin[g]; t < shard_begin[g + 1]; ++t)
            for (int32_t j = 0; j < k; ++j)
                counts[(int64_t)g * E + topk[t * k + j]] += 1;

    /* 2-3. totals over sources, expert offsets, rank offsets */
    int64_t run = 0;
    for (int32_t e = 0; e < E; ++e) {
        expert_offsets[e] = (int32_t)run;
        for (int32_t g = 0; g < G; ++g)
            run += counts[(int64_t)g * E + e];
    }
    expert_offsets[E] = (int32_t)run;
    int32_t *first = (int32_t *)malloc(sizeof(int32_t) * (size_t)(R + 1));
    int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    if (first == NULL || cursor == NULL) {
        free(first);
        free(cursor);
        return ORC_INVALID_ARG;
    }
    oracle_partition(E, R, first);
    for (int32_t r = 0; r <= R; ++r)
        rank_offsets[r] = expert_offsets[first[r]];

    /* 4-5. each source's first row per expert, then its tokens in order */
    for (int32_t g = 0; g < G; ++g) {
        for (int32_t e = 0; e < E; ++e) {
            int64_t before = 0;
            for (int32_t h = 0; h < g; ++h)
                before += counts[(int64_t)h * E + e];
            cursor[e] = (int32_t)(expert_offsets[e] + before);
        }
        for (int64_t t = shard_begin[g]; t < shard_begin[g + 1]; ++t)
            for (int32_t j = 0; j < k; ++j) {
                int32_t e = topk[t * k + j];
                slot[t * k + j] = cursor[e];
                cursor[e] += 1;
            }
    }
    free(first);
    free(cursor);
    return ORC_OK;
}

/* Inverse of the node staging map: staging row node_offsets[n] +
 * node_slot[t][n] holds token t, for every (t, n) with node_slot[t][n] >= 0.
 * node_src has node_offsets[N] entries.  (FUSCO article, section "FUSCO 的
 * 核心创新": a forwarder handles the rows staged for its node; listing them
 * row by row lets the forwarding work be divided by rows.) */
void oracle_node_sources(int64_t T, int32_t N, const int32_t *node_offsets,
                         const int32_t *node_slot, int32_t *node_src)
{
    for (int64_t t = 0; t < T; ++t)
        for (int32_t n = 0; n < N; ++n) {
            int32_t ns = node_slot[t * N + n];
            if (ns >= 0)
                node_src[(int64_t)node_offsets[n] + ns] = (int32_t)t;
        }
}

/* ------------------------------------------------------------------ */
/* Dispatch                                                            */
/* ------------------------------------------------------------------ */

/* recv[slot[t][j]] = x[t] for every (t, j).  Rows are H bf16 values. */
void oracle_dispatch_flat(int64_t T, int32_t H, int32_t k,
                          const int32_t *slot, const uint16_t *x,
                          uint16_t *recv)
{
    size_t row_bytes = sizeof(uint16_t) * (size_t)H;
    for (int64_t t = 0; t < T; ++t)
        for (int32_t j = 0; j < k; ++j) {
            int64_t dst = slot[t * k + j];
            memcpy(recv + dst * H, x + t * H, row_bytes);
        }
}

/* Two-level dispatch.  Phase 1: x[t] goes once into the staging region of
 * every node it touches (row node_offsets[n] + node_slot[t][n]).  Phase 2:
 * for each node, in node order, each staging row is copied from staging to
 * every expert row of its token that lies on that node.  A row lies on node
 * n when its receive row falls in node n's rank range
 * [rank_offsets[n*R/N], rank_offsets[(n+1)*R/N]). */
void oracle_dispatch_two_level(int64_t T, int32_t H, int32_t k, int32_t R,
                               int32_t N, const int32_t *slot,
                               const int32_t *rank_offsets,
                               const int32_t *node_offsets,
                               const int32_t *node_slot,
                               const uint16_t *x, uint16_t *staging,
                               uint16_t *recv)
{
    size_t row_bytes = sizeof(uint16_t) * (size_t)H;
    int32_t ranks_per_node = R / N;
    for (int64_t t = 0; t < T; ++t)
        for (int32_t n = 0; n < N; ++n) {
            int32_t ns = node_slot[t * N + n];
            if (ns >= 0) {
                int64_t row = (int64_t)node_offsets[n] + ns;
                memcpy(staging + row * H, x + t * H, row_bytes);
            }
        }
    for (int32_t n = 0; n < N; ++n) {
        int32_t lo = rank_offsets[n * ranks_per_node];
        int32_t hi = rank_offsets[(n + 1) * ranks_per_node];
        for (int64_t t = 0; t < T; ++t) {
            int32_t ns = node_slot[t * N + n];
            if (ns < 0)
                continue;
            int64_t srow = (int64_t)node_offsets[n] + ns;
            for (int32_t j = 0; j < k; ++j) {
                int32_t dst = slot[t * k + j];
                if (dst >= lo && dst < hi)
                    memcpy(recv + (int64_t)dst * H, staging + srow * H, row_bytes);
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* Combine                                                             */
/* ------------------------------------------------------------------ */

/* y[t][h] = bf16_rne( fma(w[t][k-1], eo[slot[t][k-1]][h], ...
 *                      fma(w[t][0], eo[slot[t][0]][h], +0.0f)) ) */
void oracle_combine(int64_t T, int32_t H, int32_t k, const int32_t *slot,
                    const float *w, const uint16_t *eo, uint16_t *y)
{
    for (int64_t t = 0; t < T; ++t)
        for (int32_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int32_t j = 0; j < k; ++j) {
                int64_t row = slot[t * k + j];
                float v = oracle_bf16_to_f32(eo[row * H + h]);
                acc = fmaf(w[t * k + j], v, acc);
            }
            y[t * H + h] = oracle_f32_to_bf16(acc);
        }
}

/* Same sum for a chosen list of tokens only; y_rows is [n_tokens][H].  Used
 * to check large workloads on sampled tokens. */
void oracle_combine_tokens(int64_t n_tokens, const int64_t *tokens,
                           int32_t H, int32_t k, const int32_t *slot,
                           const float *w, const uint16_t *eo,
                           uint16_t *y_rows)
{
    for (int64_t i = 0; i < n_tokens; ++i) {
        int64_t t = tokens[i];
        for (int32_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int32_t j = 0; j < k; ++j) {
                int64_t row = slot[t * k + j];
                float v = oracle_bf16_to_f32(eo[row * H + h]);
                acc = fmaf(w[t * k + j], v, acc);
            }
            y_rows[i * H + h] = oracle_f32_to_bf16(acc);
        }
    }
}

/* ------------------------------------------------------------------ */
/* Token loops over host threads (timing only)                         */
/* ------------------------------------------------------------------ */

/* oracle_dispatch_flat, oracle_dispatch_two_level and oracle_combine with
 * their token loops split over OpenMP threads.  Each token's rows are written
 * by one thread with exactly the arithmetic of the serial functions, so the
 * results are identical; the layout stays serial (its slot order is defined
 * by token order).  These exist to time the oracle on all host cores beside
 * the single-thread runs; the serial functions above are the reference. */
int oracle_parallel_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_dispatch_flat_par(int64_t T, int32_t H, int32_t k,
                              const int32_t *slot, const uint16_t *x,
                              uint16_t *recv)
{
    size_t bytes = sizeof(uint16_t) * (size_t)H;
#pragma omp parallel for schedule(static)
    for (int64_t tok = 0; tok < T; ++tok)
        for (int32_t col = 0; col < k; ++col)
            memcpy(recv + (int64_t)slot[tok * k + col] * H, x + tok * H, bytes);
}

void oracle_dispatch_two_level_par(int64_t T, int32_t H, int32_t k, int32_t R,
                                   int32_t N, const int32_t *slot,
                                   const int32_t *rank_offsets,
                                   const int32_t *node_offsets,
                                   const int32_t *node_slot,
                                   const uint16_t *x, uint16_t *staging,
                                   uint16_t *recv)
{
    size_t bytes = sizeof(uint16_t) * (size_t)H;
    int32_t per_node = R / N;
#pragma omp parallel for schedule(static)
    for (int64_t tok = 0; tok < T; ++tok)
        for (int32_t nd = 0; nd < N; ++nd) {
            int32_t rank_in_node = node_slot[tok * N + nd];
            if (rank_in_node < 0)
                continue;
            memcpy(staging + ((int64_t)node_offsets[nd] + rank_in_node) * H, x + tok * H, bytes);
        }
    for (int32_t nd = 0; nd < N; ++nd) {
        int32_t first = rank_offsets[nd * per_node];
        int32_t last = rank_offsets[(nd + 1) * per_node];
#pragma omp parallel for schedule(static)
        for (int64_t tok = 0; tok < T; ++tok) {
            int32_t rank_in_node = node_slot[tok * N + nd];
            if (rank_in_node < 0)
                continue;
            const uint16_t *from = staging + ((int64_t)node_offsets[nd] + rank_in_node) * H;
            for (int32_t col = 0; col < k; ++col) {
                int32_t to = slot[tok * k + col];
                if (to >= first && to < last)
                    memcpy(recv + (int64_t)to * H, from, bytes);
            }
        }
    }
}

void oracle_combine_par(int64_t T, int32_t H, int32_t k, const int32_t *slot,
                        const float *w, const uint16_t *eo, uint16_t *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t tok = 0; tok < T; ++tok)
        for (int32_t col_h = 0; col_h < H; ++col_h) {
            float sum = 0.0f;
            for (int32_t col = 0; col < k; ++col)
                sum = fmaf(w[tok * k + col],
                           oracle_bf16_to_f32(eo[(int64_t)slot[tok * k + col] * H + col_h]), sum);
            y[tok * H + col_h] = oracle_f32_to_bf16(sum);
        }
}

/* Combine in the reduce-scatter order (INC-MoE abstract: combine as a
 * ReduceScatter; TensorRT-LLM PR #13888: the AllGather + ReduceScatter
 * fallback path).  Each rank r first sums, in fp32 with one FMA per column
 * j in order, the token's expert rows that live on r (its receive rows lie in
 * [rank_offsets[r], rank_offsets[r+1])); the R partial sums are then added
 * in rank order starting from +0, and the total is rounded once to bf16. */
void oracle_combine_rank_partials(int64_t T, int32_t H, int32_t k, int32_t R,
                                  const int32_t *slot, const int32_t *rank_offsets,
                                  const float *w, const uint16_t *eo, uint16_t *y)
{
    for (int64_t t = 0; t < T; ++t)
        for (int32_t h = 0; h < H; ++h) {
            float total = 0.0f;
            for (int32_t r = 0; r < R; ++r) {
                float part = 0.0f;
                for (int32_t j = 0; j < k; ++j) {
                    int32_t row = slot[t * k + j];
                    if (row >= rank_offsets[r] && row < rank_offsets[r + 1])
                        part = fmaf(w[t * k + j], oracle_bf16_to_f32(eo[(int64_t)row * H + h]), part);
                }
                total = total + part;
            }
            y[t * H + h] = oracle_f32_to_bf16(total);
        }
}

/* ------------------------------------------------------------------ */
/* FP8 (e4m3) payload                                                  */
/* ------------------------------------------------------------------ */
/* TensorRT-LLM PR #13888 (the ConfigurableMoE commit) validates an fp8
 * low-precision combine at rtol 0.02 / atol 0.15.  The encoding is the OCP
 * FP8 E4M3 format: sign, 4 exponent bits (bias 7), 3 mantissa bits, no
 * infinities, S.1111.111 is NaN, largest finite value 448.  The reading
 * taken for the payload: one fp32 scale per row, scale = amax / 448 (amax =
 * largest |value| of the row; a zero row uses scale 1), values stored as
 * e4m3(v * (448 / amax)) rounded to nearest even and saturated to +-448. */

/* Decode one e4m3 code (exact in fp32). */
float oracle_e4m3_to_f32(uint8_t c)
{
    int sign = (c >> 7) & 1;
    int exp_bits = (c >> 3) & 0xF;
    int man = c & 7;
    float v;
    if (exp_bits == 0xF && man == 7)
        return sign ? -NAN : NAN;
    if (exp_bits == 0)
        v = ldexpf((float)man, -9);                 /* subnormal: m/8 * 2^-6 */
    else
        v = ldexpf((float)(8 + man), exp_bits - 10); /* (1 + m/8) * 2^(e-7) */
    return sign ? -v : v;
}

/* Encode: round to nearest (ties to even code) over the finite e4m3 values,
 * saturating beyond 448; NaN maps to the NaN code.  The 127 non-negative
 * finite codes decode to increasing values, so the code just below |f| is
 * found by binary search over their decoded values. */
static float e4m3_value[127];
static int e4m3_value_ready = 0;

uint8_t oracle_f32_to_e4m3(float f)
{
    if (!e4m3_value_ready) {
        for (int c = 0; c < 127; ++c)
            e4m3_value[c] = oracle_e4m3_to_f32((uint8_t)c);
        e4m3_value_ready = 1;
    }
    if (f != f)
        return 0x7F;
    uint8_t sign = signbit(f) ? 0x80 : 0x00;
    float a = fabsf(f);
    if (a >= 448.0f)
        return (uint8_t)(sign | 0x7E);
    int lo = 0, hi = 126;            /* invariant: value[lo] <= a < value[hi] */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (e4m3_value[mid] <= a)
            lo = mid;
        else
            hi = mid;
    }
    double dlo = (double)a - (double)e4m3_value[lo], dhi = (double)e4m3_value[hi] - (double)a;
    int pick;
    if (dlo < dhi)
        pick = lo;
    else if (dhi < dlo)
        pick = hi;
    else
        pick = (lo & 1) ? hi : lo;   /* tie: even code */
    return (uint8_t)(sign | pick);
}

void oracle_e4m3_to_f32_array(const uint8_t *src, float *dst, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = oracle_e4m3_to_f32(src[i]);
}

void oracle_f32_to_e4m3_array(const float *src, uint8_t *dst, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = oracle_f32_to_e4m3(src[i]);
}

/* Quantize `rows` bf16 rows of H values to e4m3 with one scale per row. */
void oracle_quantize_rows_fp8(int64_t rows, int32_t H, const uint16_t *src, uint8_t *q,
                              float *scale)
{
    for (int64_t r = 0; r < rows; ++r) {
        float amax = 0.0f;
        for (int32_t h = 0; h < H; ++h) {
            float v = fabsf(oracle_bf16_to_f32(src[r * H + h]));
            if (v > amax)
                amax = v;
        }
        float inv = amax > 0.0f ? 448.0f / amax : 1.0f;
        scale[r] = amax > 0.0f ? amax / 448.0f : 1.0f;
        for (int32_t h = 0; h < H; ++h)
            q[r * H + h] = oracle_f32_to_e4m3(oracle_bf16_to_f32(src[r * H + h]) * inv);
    }
}

/* fp8 dispatch: quantize x, then every destination row receives the token's
 * codes and scale. */
void oracle_dispatch_fp8(int64_t T, int32_t H, int32_t k, const int32_t *slot,
                         const uint16_t *x, uint8_t *recv_q, float *recv_scale)
{
    uint8_t *qt = (uint8_t *)malloc((size_t)H);
    float st;
    for (int64_t t = 0; t < T; ++t) {
        oracle_quantize_rows_fp8(1, H, x + t * H, qt, &st);
        for (int32_t j = 0; j < k; ++j) {
            int64_t dst = slot[t * k + j];
            memcpy(recv_q + dst * H, qt, (size_t)H);
            recv_scale[dst] = st;
        }
    }
    free(qt);
}

/* fp8 combine: coef_j = w[t][j] * scale[slot[t][j]] (fp32), then
 * acc = fma(coef_j, e4m3(eo_q[slot][h]), acc) for j = 0..k-1 from +0, one
 * bf16 rounding. */
void oracle_combine_fp8(int64_t T, int32_t H, int32_t k, const int32_t *slot,
                        const float *w, const uint8_t *eo_q, const float *eo_scale,
                        uint16_t *y)
{
    for (int64_t t = 0; t < T; ++t)
        for (int32_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int32_t j = 0; j < k; ++j) {
                int64_t row = slot[t * k + j];
                float coef = w[t * k + j] * eo_scale[row];
                acc = fmaf(coef, oracle_e4m3_to_f32(eo_q[row * H + h]), acc);
            }
            y[t * H + h] = oracle_f32_to_bf16(acc);
        }
}

/*
 * moe_oracle.c -- plain, slow CPU oracle for MoE token dispatch and combine.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker, not the product: only
 * the test suite, the package's smoke check and the benchmark's CPU-baseline
 * leg may load it.  It shares no code, header, table or constant with the
 * CUDA library; the status bit values below are this file's own copy of the
 * documented contract.
 *
 * Every routine uses plain loops and does its floating point in fp64 unless a
 * rounding step is part of the definition.  The plain build (no -fopenmp) is
 * single-threaded and is the checker.  A second build of this same file with
 * -fopenmp serves only as the multi-core CPU baseline: its pragmas split
 * loops whose iterations are independent (each writes its own outputs and
 * the status bits are OR-reduced), so both builds give identical results.
 * Sources:
 *
 *  [DeepEP-272]  DeepEP issue "Does Deepep's Dispatch/Combine Support Autograd
 *                Like PyTorch's all_to_all?" -- get_dispatch_layout outputs
 *                (num_tokens_per_rank, num_tokens_per_expert,
 *                is_token_in_rank); dispatch backward is a combine.
 *  [DS-8847]     DeepSpeed PR "AutoEP: support combine_impl=fused_weighted_sum
 *                with AutoEP+AutoTP folding", sections Problem / Change /
 *                Benchmark -- flat index token*top_k+slot, router-dtype
 *                weights scattered to [tokens, top_k], FP32 accumulation,
 *                coverage RuntimeError, row and score gradients.
 *  [DS-AutoEP]   DeepSpeed AutoEP base PR, sections Attribution and Design --
 *                reorder tokens by expert, token-group alignment / padding
 *                for grouped GEMM, restore the original token order.
 *  [DS-8190]     DeepSpeed PR "Derive AutoEP rank splits from the per-expert
 *                count exchange", sections Redundancy and Fix -- the count
 *                matrix [ep_size, E_local], input_splits = its row sums, and
 *                received_counts.sum(dim=1) == output_splits.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - padding: an expert with c tokens occupies ceil(c/align)*align rows, so an
 *    empty expert occupies none;
 *  - order inside an expert's group: stable by flat index (token, then slot);
 *  - logical ranks: source rank s owns tokens [s*T/R, (s+1)*T/R), destination
 *    rank r owns experts [r*E/R, (r+1)*E/R);
 *  - an out-of-range expert id (including -1) is an error: the assignment is
 *    skipped and the EXPERT_OOR bit is returned;
 *  - pad rows are zero, rows past the padded total are left untouched and
 *    carry row_to_flat = -1;
 *  - the FP32 combine is an fmaf chain over slots k = 0..K-1 from 0 with one
 *    round-to-nearest-even to bf16 (reported by out_seq); the fp64 sum is the
 *    reference value the tolerance is measured against;
 *  - grad_w is accumulated in fp64 (bf16 x bf16 products are exact).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Threads the loops below may use: 1 in the plain build. */
int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Status bits (the library's documented values; this file's own copy). */
#define ORC_EXPERT_OOR 1
#define ORC_CAPACITY 2
#define ORC_ROW_OOR 4
#define ORC_COVERAGE 8

/* ---------------------------------------------------------------- bf16 --- */

/* bfloat16 is the top 16 bits of an IEEE binary32.  Round to nearest, ties to
 * even, from the definition: keep the top half; look at the discarded low
 * half; above the midpoint round up, below it keep, exactly at it round up
 * only when the kept value is odd.  Rounding up is +1 on the kept bits, which
 * carries into the exponent (and to infinity) as IEEE ordering requires.
 * NaN stays NaN (quiet bit forced). */
uint16_t oracle_bf16_from_float(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t kept = u >> 16;
    uint32_t low = u & 0xffffu;
    if (low > 0x8000u || (low == 0x8000u && (kept & 1u))) kept += 1u;
    return (uint16_t)kept;
}

float oracle_float_from_bf16(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Element-wise helpers so tests can pin the rounding against a library. */
void oracle_bf16_round_array(const float* in, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_from_float(in[i]);
}

/* -------------------------------------------------------------- layout --- */

/* get_dispatch_layout [DeepEP-272] plus the count matrix of [DS-8190] and the
 * padded group offsets of [DS-AutoEP] (alignment / padding helpers).
 *
 *   tokens_per_expert[e]        = #{(t,k) : topk_idx[t,k] = e}
 *   counts[s][r][el]            = #{(t,k) : t in block s, topk_idx[t,k] = r*El+el}
 *   splits[s][r]                = sum over el of counts[s][r][el]
 *                                 (row s = input_splits of source rank s)
 *   is_token_in_rank[t][r]      = 1 if some slot of t routes to an expert of r
 *   tokens_per_rank[s][r]       = #{t in block s : is_token_in_rank[t][r]}
 *   offsets[0] = 0, offsets[e+1] = offsets[e] + ceil(c_e/align)*align
 *
 * Returns status bits (ORC_EXPERT_OOR if some id is outside [0, E)). */
int oracle_layout(const int64_t* topk_idx, int T, int K, int E, int R, int align,
                  int32_t* tokens_per_expert, int32_t* counts, int32_t* splits,
                  int32_t* tokens_per_rank, uint8_t* is_token_in_rank,
                  int32_t* offsets) {
    int status = 0;
    int El = E / R;
    int Tb = T / R;
    memset(tokens_per_expert, 0, sizeof(int32_t) * (size_t)E);
    memset(counts, 0, sizeof(int32_t) * (size_t)R * (size_t)E);
    memset(splits, 0, sizeof(int32_t) * (size_t)R * (size_t)R);
    memset(tokens_per_rank, 0, sizeof(int32_t) * (size_t)R * (size_t)R);
    memset(is_token_in_rank, 0, (size_t)T * (size_t)R);

    for (int t = 0; t < T; ++t) {
        int s = t / Tb;
        for (int k = 0; k < K; ++k) {
            int64_t e = topk_idx[(int64_t)t * K + k];
            if (e < 0 || e >= E) {
                status |= ORC_EXPERT_OOR;
                continue;
            }
            int r = (int)(e / El);
            int el = (int)(e % El);
            tokens_per_expert[e] += 1;
            counts[((int64_t)s * R + r) * El + el] += 1;
            is_token_in_rank[(int64_t)t * R + r] = 1;
        }
    }
    for (int s = 0; s < R; ++s)
        for (int r = 0; r < R; ++r) {
            int32_t sum = 0;
            for (int el = 0; el < El; ++el) sum += counts[((int64_t)s * R + r) * El + el];
            splits[s * R + r] = sum;
        }
    for (int t = 0; t < T; ++t) {
        int s = t / Tb;
        for (int r = 0; r < R; ++r) tokens_per_rank[s * R + r] += is_token_in_rank[(int64_t)t * R + r];
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) {
        int32_t c = tokens_per_expert[e];
        int32_t padded = ((c + align - 1) / align) * align;
        offsets[e + 1] = offsets[e] + padded;
    }
    return status;
}

/* output_splits of every destination rank, counted directly: the number of
 * assignments source block s sends to rank r, i.e. what the per-rank-total
 * exchange of [DS-8190] (Redundancy, "exchange 1") would have delivered.
 * Independent of the count matrix, so that received_counts.sum(dim=1) ==
 * output_splits can be checked against it.  out[r][s]. */
void oracle_output_splits(const int64_t* topk_idx, int T, int K, int E, int R, int32_t* out) {
    int El = E / R;
    int Tb = T / R;
    for (int r = 0; r < R; ++r)
        for (int s = 0; s < R; ++s) {
            int32_t n = 0;
            for (int t = s * Tb; t < (s + 1) * Tb; ++t)
                for (int k = 0; k < K; ++k) {
                    int64_t e = topk_idx[(int64_t)t * K + k];
                    if (e >= (int64_t)r * El && e < (int64_t)(r + 1) * El) ++n;
                }
            out[r * R + s] = n;
        }
}

/* Row bases of expert parallelism without a send buffer ([DS-8190]
 * Redundancy: each source rank s knows its assignments to every expert, and
 * the matrix of those counts over the ranks fixes where every rank's rows go;
 * [DS-AutoEP] Attribution: group alignment for the grouped GEMM).  The
 * receive buffer of owner rank r holds its experts [r*El, (r+1)*El) in
 * order, each expert's group padded to a multiple of align, and inside a
 * group the rows of source rank 0 first, then rank 1, and so on.  From
 * all_counts [R][E] (row s = the per-expert counts of source rank s):
 *
 *   own_counts[el]  = sum over s of all_counts[s][rank*El + el]
 *   own_offsets[el] = padded start of group el in rank `rank`'s buffer,
 *   own_offsets[El] = that buffer's padded total
 *   dest_base[e]    = padded start of e's group in its owner's buffer
 *                     + sum over s < rank of all_counts[s][e]
 *   max_rows        = the largest padded total over the owners
 *
 * Returns ORC_COVERAGE (and treats the count as 0) for a negative count. */
int oracle_rank_bases(const int32_t* all_counts, int R, int E, int rank, int align,
                      int32_t* dest_base, int32_t* own_offsets, int32_t* own_counts,
                      int32_t* max_rows) {
    int status = 0;
    int El = E / R;
    int64_t best = 0;
    for (int r = 0; r < R; ++r) {
        int64_t start = 0;   /* running padded start inside owner r's buffer */
        for (int el = 0; el < El; ++el) {
            int e = r * El + el;
            int64_t total = 0, before = 0;
            for (int s = 0; s < R; ++s) {
                int64_t c = all_counts[(int64_t)s * E + e];
                if (c < 0) {
                    status |= ORC_COVERAGE;
                    c = 0;
                }
                total += c;
                if (s < rank) before += c;
            }
            dest_base[e] = (int32_t)(start + before);
            if (r == rank) {
                own_offsets[el] = (int32_t)start;
                own_counts[el] = (int32_t)total;
            }
            start += ((total + align - 1) / align) * align;
        }
        if (r == rank) own_offsets[El] = (int32_t)start;
        if (start > best) best = start;
    }
    *max_rows = (int32_t)best;
    return status;
}

/* ------------------------------------------------------------- permute --- */

typedef struct {
    int32_t expert;
    int32_t flat;
} orc_assign;

static int orc_cmp_assign(const void* a, const void* b) {
    const orc_assign* x = (const orc_assign*)a;
    const orc_assign* y = (const orc_assign*)b;
    if (x->expert != y->expert) return x->expert < y->expert ? -1 : 1;
    if (x->flat != y->flat) return x->flat < y->flat ? -1 : 1;
    return 0;
}

/* Reorder token rows by expert ([DS-AutoEP] runtime step 3; [DeepEP-272]
 * dispatch on one device).  Assignments are sorted by the key (expert, flat
 * index f = t*K + k) with the C library sort; the i-th assignment of expert e
 * in that order lands on row offsets[e] + i.
 *
 *   x_perm[row(f)] = x[t]          flat_to_row[f] = row(f)
 *   row_to_flat[row(f)] = f        all other rows: row_to_flat = -1
 *   pad rows [offsets[e] + c_e, offsets[e+1]) are zero when zero_pad != 0;
 *   rows [offsets[E], N_cap) keep their contents.
 *
 * Rows at or past N_cap are not written (ORC_CAPACITY). */
int oracle_permute(const uint16_t* x, const int64_t* topk_idx, int T, int K, int E, int H,
                   const int32_t* offsets, int zero_pad, int64_t N_cap, uint16_t* x_perm,
                   int32_t* row_to_flat, int32_t* flat_to_row) {
    int status = 0;
    int64_t A = (int64_t)T * K;
    orc_assign* list = (orc_assign*)malloc(sizeof(orc_assign) * (size_t)(A > 0 ? A : 1));
    int64_t n = 0;
    for (int64_t f = 0; f < A; ++f) {
        flat_to_row[f] = -1;
        int64_t e = topk_idx[f];
        if (e < 0 || e >= E) {
            status |= ORC_EXPERT_OOR;
            continue;
        }
        list[n].expert = (int32_t)e;
        list[n].flat = (int32_t)f;
        ++n;
    }
    qsort(list, (size_t)n, sizeof(orc_assign), orc_cmp_assign);

#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < N_cap; ++row) row_to_flat[row] = -1;
    if ((int64_t)offsets[E] > N_cap) status |= ORC_CAPACITY;

    int64_t i = 0;
    while (i < n) {
        int32_t e = list[i].expert;
        int64_t j = i;
        while (j < n && list[j].expert == e) {
            int64_t row = (int64_t)offsets[e] + (j - i);
            int32_t f = list[j].flat;
            if (row < N_cap) {
                int64_t t = f / K;
                memcpy(x_perm + row * H, x + t * H, sizeof(uint16_t) * (size_t)H);
                row_to_flat[row] = f;
                flat_to_row[f] = (int32_t)row;
            } else {
                status |= ORC_CAPACITY;
            }
            ++j;
        }
        i = j;
    }
    if (zero_pad) {
        int64_t end = (int64_t)offsets[E] < N_cap ? (int64_t)offsets[E] : N_cap;
#pragma omp parallel for schedule(static)
        for (int64_t row = 0; row < end; ++row)
            if (row_to_flat[row] < 0) memset(x_perm + row * H, 0, sizeof(uint16_t) * (size_t)H);
    }
    free(list);
    return status;
}

/* Dispatch of an arbitrary row payload ([DeepEP-272]: dispatch takes x as a
 * bf16 tensor or as an FP8 tuple (data, scales); [DS-8847] Tests: fp32 and
 * bf16 rows).  The rows are opaque bytes: every token row of x is row_bytes
 * bytes and, when aux != NULL, every token also owns an aux row of aux_bytes
 * bytes (the FP8 scales), which travels with it.  The destination row of
 * each assignment is the one oracle_permute defines -- the i-th assignment
 * of expert e in (expert, flat index) order lands on offsets[e] + i -- found
 * here with the same sort:
 *
 *   x_perm[row(f)] = x[t]     aux_perm[row(f)] = aux[t]
 *   maps, pad rows (zero, both payloads, when zero_pad) and the untouched
 *   tail exactly as in oracle_permute. */
int oracle_permute_payload(const uint8_t* x, int64_t row_bytes, const uint8_t* aux,
                           int64_t aux_bytes, const int64_t* topk_idx, int T, int K, int E,
                           const int32_t* offsets, int zero_pad, int64_t N_cap, uint8_t* x_perm,
                           uint8_t* aux_perm, int32_t* row_to_flat, int32_t* flat_to_row) {
    int status = 0;
    int64_t A = (int64_t)T * K;
    orc_assign* list = (orc_assign*)malloc(sizeof(orc_assign) * (size_t)(A > 0 ? A : 1));
    int64_t n = 0;
    for (int64_t f = 0; f < A; ++f) {
        flat_to_row[f] = -1;
        int64_t e = topk_idx[f];
        if (e < 0 || e >= E) {
            status |= ORC_EXPERT_OOR;
            continue;
        }
        list[n].expert = (int32_t)e;
        list[n].flat = (int32_t)f;
        ++n;
    }
    qsort(list, (size_t)n, sizeof(orc_assign), orc_cmp_assign);
    for (int64_t row = 0; row < N_cap; ++row) row_to_flat[row] = -1;
    if ((int64_t)offsets[E] > N_cap) status |= ORC_CAPACITY;

    int64_t first = 0;   /* index in `list` of the current expert's first assignment */
    for (int64_t i = 0; i < n; ++i) {
        if (i == 0 || list[i].expert != list[i - 1].expert) first = i;
        int32_t e = list[i].expert;
        int64_t row = (int64_t)offsets[e] + (i - first);
        int32_t f = list[i].flat;
        if (row >= N_cap) {
            status |= ORC_CAPACITY;
            continue;
        }
        int64_t t = f / K;
        memcpy(x_perm + row * row_bytes, x + t * row_bytes, (size_t)row_bytes);
        if (aux) memcpy(aux_perm + row * aux_bytes, aux + t * aux_bytes, (size_t)aux_bytes);
        row_to_flat[row] = f;
        flat_to_row[f] = (int32_t)row;
    }
    if (zero_pad) {
        for (int64_t row = 0; row < (int64_t)offsets[E] && row < N_cap; ++row)
            if (row_to_flat[row] < 0) {
                memset(x_perm + row * row_bytes, 0, (size_t)row_bytes);
                if (aux) memset(aux_perm + row * aux_bytes, 0, (size_t)aux_bytes);
            }
    }
    free(list);
    return status;
}

/* The definition of the row written for assignment f, counted by brute force
 * in O(A^2): row(f) = offsets[e] + #{f' < f : topk_idx[f'] = e}.  Used only to
 * pin oracle_permute on small inputs. */
void oracle_bruteforce_rows(const int64_t* topk_idx, int T, int K, int E, const int32_t* offsets,
                            int32_t* rows) {
    int64_t A = (int64_t)T * K;
    for (int64_t f = 0; f < A; ++f) {
        int64_t e = topk_idx[f];
        if (e < 0 || e >= E) {
            rows[f] = -1;
            continue;
        }
        int32_t before = 0;
        for (int64_t g = 0; g < f; ++g)
            if (topk_idx[g] == e) ++before;
        rows[f] = offsets[e] + before;
    }
}

/* ------------------------------------------------------ stand-in expert --- */

/* The seeded per-expert stand-in y = x * s_e that sits where the grouped
 * expert MLP would: every real row of expert e becomes
 * bf16_rn(fp32(x) * s_e) -- the product of a bf16 and an fp32 is exact in
 * fp64, rounded once to fp32 and then once to bf16.  Pad rows of expert e
 * are written as zero; rows past offsets[E] are untouched. */
void oracle_expert_scale(const uint16_t* rows, const int32_t* offsets,
                         const int32_t* tokens_per_expert, int E, int H, const float* scales,
                         uint16_t* out) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int e = 0; e < E; ++e) {
        int64_t begin = offsets[e];
        int64_t real_end = begin + tokens_per_expert[e];
        int64_t end = offsets[e + 1];
        double s = (double)scales[e];
        for (int64_t row = begin; row < end; ++row)
            for (int h = 0; h < H; ++h) {
                int64_t idx = row * H + h;
                if (row < real_end) {
                    double p = (double)oracle_float_from_bf16(rows[idx]) * s;
                    out[idx] = oracle_bf16_from_float((float)p);
                } else {
                    out[idx] = 0;
                }
            }
    }
}

/* ------------------------------------------------------------- combine --- */

/* fused_weighted_restore [DS-8847] (Change; Benchmark): for every token t,
 *
 *   out[t] = sum_{k=0}^{K-1} w[t,k] * rows[flat_to_row[t*K+k]]
 *
 * with weights in the router dtype (passed here widened to float, which is
 * exact for fp32 and bf16), or all ones when w == NULL (dispatch backward is
 * a combine, [DeepEP-272]).  out_ref receives the fp64 sum (products are
 * exact in fp64).  out_seq, when not NULL, receives the FP32 reading: acc = 0,
 * then acc = fmaf(w, y, acc) for k = 0..K-1 in order, then one RNE to bf16.
 * A slot whose row lies outside [0, N_cap) contributes nothing and sets
 * ORC_ROW_OOR. */
int oracle_combine(const uint16_t* rows, int64_t N_cap, const int32_t* flat_to_row,
                   const float* w, int T, int K, int H, double* out_ref, uint16_t* out_seq) {
    int status = 0;
#pragma omp parallel for reduction(|: status) schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int h = 0; h < H; ++h) {
            double sum = 0.0;
            float acc = 0.0f;
            for (int k = 0; k < K; ++k) {
                int64_t f = (int64_t)t * K + k;
                int64_t row = flat_to_row[f];
                if (row < 0 || row >= N_cap) {
                    status |= ORC_ROW_OOR;
                    continue;
                }
                float wk = w ? w[f] : 1.0f;
                float y = oracle_float_from_bf16(rows[row * H + h]);
                sum += (double)wk * (double)y;
                acc = fmaf(wk, y, acc);
            }
            out_ref[(int64_t)t * H + h] = sum;
            if (out_seq) out_seq[(int64_t)t * H + h] = oracle_bf16_from_float(acc);
        }
    }
    return status;
}

/* fused_weighted_restore on fp32 rows ([DS-8847] Tests: "fp32 and bf16
 * rows"; the activation dtype is fp32, so the output is fp32 and the FP32
 * accumulation is not followed by a narrower rounding).  out_ref receives
 * the fp64 sum (a product of two floats is exact in fp64); out_seq, when not
 * NULL, the FP32 reading: acc = 0, acc = fmaf(w, y, acc) for k = 0..K-1 in
 * order, stored as is.  Out-of-range slots as in oracle_combine. */
int oracle_combine_f32(const float* rows, int64_t N_cap, const int32_t* flat_to_row,
                       const float* w, int T, int K, int H, double* out_ref, float* out_seq) {
    int status = 0;
#pragma omp parallel for reduction(|: status) schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int h = 0; h < H; ++h) {
            double sum = 0.0;
            float acc = 0.0f;
            for (int k = 0; k < K; ++k) {
                int64_t f = (int64_t)t * K + k;
                int64_t row = flat_to_row[f];
                if (row < 0 || row >= N_cap) {
                    status |= ORC_ROW_OOR;
                    continue;
                }
                float wk = w ? w[f] : 1.0f;
                float y = rows[row * H + h];
                sum += (double)wk * (double)y;
                acc = fmaf(wk, y, acc);
            }
            out_ref[(int64_t)t * H + h] = sum;
            if (out_seq) out_seq[(int64_t)t * H + h] = acc;
        }
    }
    return status;
}

/* Coverage validation [DS-8847] (Change: "raises a clear RuntimeError if the
 * gathered rows do not cover every (token, slot)"): every flat index f in
 * [0, A) must be held by exactly one row.  Checked as the two maps being
 * mutual inverses: row_to_flat[flat_to_row[f]] == f for every f, and
 * flat_to_row[row_to_flat[r]] == r for every row r with row_to_flat[r] >= 0.
 * Returns ORC_COVERAGE when either fails. */
int oracle_check_coverage(const int32_t* row_to_flat, const int32_t* flat_to_row, int64_t N_cap,
                          int64_t A) {
    for (int64_t f = 0; f < A; ++f) {
        int64_t row = flat_to_row[f];
        if (row < 0 || row >= N_cap) return ORC_COVERAGE;
        if (row_to_flat[row] != f) return ORC_COVERAGE;
    }
    for (int64_t row = 0; row < N_cap; ++row) {
        int64_t f = row_to_flat[row];
        if (f < 0) continue;
        if (f >= A) return ORC_COVERAGE;
        if (flat_to_row[f] != row) return ORC_COVERAGE;
    }
    return 0;
}

/* Folded restore, scatter step [DS-8847] (Change: "all-gathers one flat
 * index (token * top_k + slot) ... scatters them into [tokens, top_k]" and
 * "raises a clear RuntimeError if the gathered rows do not cover every
 * (token, slot)"): given the flat index held by each gathered row (-1 for a
 * row holding none), flat_to_row[f] = the row holding f.  Every f in [0, A)
 * must be held by exactly one row; a missing f, an f held twice, or an index
 * outside [-1, A) returns ORC_COVERAGE (flat_to_row is then -1 where no row,
 * or the first row, holds f). */
int oracle_scatter_flat_index(const int32_t* row_flat, int64_t N, int64_t A, int32_t* flat_to_row) {
    int status = 0;
    for (int64_t f = 0; f < A; ++f) flat_to_row[f] = -1;
    for (int64_t row = 0; row < N; ++row) {
        int64_t f = row_flat[row];
        if (f == -1) continue;
        if (f < 0 || f >= A) {
            status |= ORC_COVERAGE;
            continue;
        }
        if (flat_to_row[f] >= 0) {
            status |= ORC_COVERAGE;
            continue;
        }
        flat_to_row[f] = (int32_t)row;
    }
    for (int64_t f = 0; f < A; ++f)
        if (flat_to_row[f] < 0) status |= ORC_COVERAGE;
    return status;
}

/* ---------------------------------------------------- combine backward --- */

/* The backward of fused_weighted_restore [DS-8847] (Tests: "row and score
 * gradients"; Benchmark: score gradient in FP32).  With g = dL/d out:
 *
 *   grad_rows[flat_to_row[f]] = bf16_rn(fp32(w[f] * g[t]))
 *   grad_w[f] = sum_h g[t,h] * rows[flat_to_row[f], h]       (fp64 sum)
 *
 * grad_w may be NULL.  When zero_pad != 0, every row below offsets[E] whose
 * row_to_flat is negative (a pad row) is written as zero; rows at or past
 * offsets[E] are untouched. */
int oracle_combine_backward(const uint16_t* g, const uint16_t* rows, int64_t N_cap,
                            const int32_t* row_to_flat, const int32_t* flat_to_row,
                            const float* w, int T, int K, int H, const int32_t* offsets, int E,
                            int zero_pad, uint16_t* grad_rows, double* grad_w) {
    int status = 0;
#pragma omp parallel for reduction(|: status) schedule(static)
    for (int t = 0; t < T; ++t)
        for (int k = 0; k < K; ++k) {
            int64_t f = (int64_t)t * K + k;
            int64_t row = flat_to_row[f];
            if (row < 0 || row >= N_cap) {
                status |= ORC_ROW_OOR;
                if (grad_w) grad_w[f] = 0.0;
                continue;
            }
            double wk = (double)w[f];
            double dot = 0.0;
            for (int h = 0; h < H; ++h) {
                double gv = (double)oracle_float_from_bf16(g[(int64_t)t * H + h]);
                double yv = (double)oracle_float_from_bf16(rows[row * H + h]);
                grad_rows[row * H + h] = oracle_bf16_from_float((float)(wk * gv));
                dot += gv * yv;
            }
            if (grad_w) grad_w[f] = dot;
        }
    if (zero_pad) {
        int64_t end = (int64_t)offsets[E] < N_cap ? (int64_t)offsets[E] : N_cap;
#pragma omp parallel for schedule(static)
        for (int64_t row = 0; row < end; ++row)
            if (row_to_flat[row] < 0) memset(grad_rows + row * H, 0, sizeof(uint16_t) * (size_t)H);
    }
    return status;
}

/* Backward of the fp32-row restore ([DS-8847] Tests): with g = grad_out,
 *
 *   grad_rows[flat_to_row[f]] = fp32(w[f] * g[t])    (the product is exact in
 *                                                     fp64, rounded once)
 *   grad_w[f] = sum_h g[t,h] * rows[flat_to_row[f], h]           (fp64 sum)
 *
 * Pad rows and out-of-range slots as in oracle_combine_backward. */
int oracle_combine_backward_f32(const float* g, const float* rows, int64_t N_cap,
                                const int32_t* row_to_flat, const int32_t* flat_to_row,
                                const float* w, int T, int K, int H, const int32_t* offsets,
                                int E, int zero_pad, float* grad_rows, double* grad_w) {
    int status = 0;
#pragma omp parallel for reduction(|: status) schedule(static)
    for (int t = 0; t < T; ++t)
        for (int k = 0; k < K; ++k) {
            int64_t f = (int64_t)t * K + k;
            int64_t row = flat_to_row[f];
            if (row < 0 || row >= N_cap) {
                status |= ORC_ROW_OOR;
                if (grad_w) grad_w[f] = 0.0;
                continue;
            }
            double wk = (double)w[f];
            double dot = 0.0;
            for (int h = 0; h < H; ++h) {
                double gv = (double)g[(int64_t)t * H + h];
                double yv = (double)rows[row * H + h];
                grad_rows[row * H + h] = (float)(wk * gv);
                dot += gv * yv;
            }
            if (grad_w) grad_w[f] = dot;
        }
    if (zero_pad) {
        int64_t end = (int64_t)offsets[E] < N_cap ? (int64_t)offsets[E] : N_cap;
#pragma omp parallel for schedule(static)
        for (int64_t row = 0; row < end; ++row)
            if (row_to_flat[row] < 0) memset(grad_rows + row * H, 0, sizeof(float) * (size_t)H);
    }
    return status;
}

/* The default folded restore of [DS-8847] (Problem: restore_combined casts
 * the routing weights to the activation dtype and runs one index_add_ per
 * top-k slot in bf16; Benchmark: its errors against FP64 and its score
 * gradient "through bf16 weights"), kept only as an accuracy comparison for
 * the fused restore.  Every product and every top-k addition is rounded to
 * bf16; each operation is carried out in fp32 and rounded once (RNE), the way
 * bf16 tensor arithmetic is:
 *
 *   wb = bf16(w);  acc = 0;
 *   for k = 0..K-1:  acc = bf16(acc + bf16(wb[t,k] * y[row(t,k)]))
 *
 * and, when g != NULL, the score gradient through the bf16 weights:
 *
 *   grad_w[t,k] = bf16( sum_h bf16(g[t,h] * y[row(t,k),h]) )   (sum in fp64)
 *
 * Out-of-range slots contribute nothing (ORC_ROW_OOR); their gradient is 0. */
int oracle_restore_activation_dtype(const uint16_t* rows, int64_t N_cap, const int32_t* flat_to_row,
                                    const float* w, const uint16_t* g, int T, int K, int H,
                                    uint16_t* out, uint16_t* grad_w) {
    int status = 0;
    for (int t = 0; t < T; ++t) {
        for (int h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int k = 0; k < K; ++k) {
                int64_t f = (int64_t)t * K + k;
                int64_t row = flat_to_row[f];
                if (row < 0 || row >= N_cap) {
                    status |= ORC_ROW_OOR;
                    continue;
                }
                float wb = oracle_float_from_bf16(oracle_bf16_from_float(w[f]));
                float y = oracle_float_from_bf16(rows[row * H + h]);
                float p = oracle_float_from_bf16(oracle_bf16_from_float(wb * y));
                acc = oracle_float_from_bf16(oracle_bf16_from_float(acc + p));
            }
            out[(int64_t)t * H + h] = oracle_bf16_from_float(acc);
        }
        if (!g || !grad_w) continue;
        for (int k = 0; k < K; ++k) {
            int64_t f = (int64_t)t * K + k;
            int64_t row = flat_to_row[f];
            if (row < 0 || row >= N_cap) {
                grad_w[f] = 0;
                continue;
            }
            double sum = 0.0;
            for (int h = 0; h < H; ++h) {
                float gv = oracle_float_from_bf16(g[(int64_t)t * H + h]);
                float yv = oracle_float_from_bf16(rows[row * H + h]);
                sum += (double)oracle_float_from_bf16(oracle_bf16_from_float(gv * yv));
            }
            grad_w[f] = oracle_bf16_from_float((float)sum);
        }
    }
    return status;
}


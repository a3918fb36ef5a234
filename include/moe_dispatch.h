/*
 * moe_dispatch.h -- C ABI of libmoe_dispatch.so: Mixture-of-Experts token
 * dispatch and combine on one NVIDIA B200 (sm_100a).
 *
 * The path, in call order (forward, then backward):
 *
 *   moe_dispatch_layout   routing layout from topk_idx           (integer)
 *   moe_permute           token rows -> expert-grouped buffer    (byte copy)
 *   moe_expert_scale      stand-in expert y = x * s_e            (fp32, one rounding)
 *   moe_combine_weighted  weighted top-k gather-sum -> tokens    (fp32 accumulate)
 *   moe_combine_backward  row gradients + routing-weight grads   (fp32 / fp64)
 *   moe_combine_weighted  with weights = NULL: dispatch backward (fp32 accumulate)
 *
 * Variants and helpers: moe_dispatch_layout_noalloc (no workspace argument),
 * moe_permute_payload (FP8 (data, scales) or any row payload),
 * moe_combine_weighted_f32 / moe_combine_backward_f32 (fp32 rows),
 * moe_scatter_flat_index (the folded restore's scatter), moe_segment_labels
 * (the receive side of expert parallelism across ranks), moe_rank_bases,
 * moe_permute_to_ranks and moe_combine_from_ranks (the row bases of, and
 * dispatch into / combine out of, the ranks' buffers directly, through peer
 * pointers).
 *
 * Sources (titles of the pages that define the operations):
 *   [DeepEP-272] DeepEP issue "Does Deepep's Dispatch/Combine Support Autograd
 *                Like PyTorch's all_to_all?": get_dispatch_layout and its
 *                outputs; the backward of dispatch is a combine and the
 *                backward of combine is a dispatch; the handle; a worst-case
 *                size instead of a CPU wait (num_worst_tokens).
 *   [DS-8847]    DeepSpeed PR "AutoEP: support combine_impl=fused_weighted_sum
 *                with AutoEP+AutoTP folding", sections Problem, Change, Tests,
 *                Benchmark: fused_weighted_restore, flat index token*top_k +
 *                slot, router-dtype weights as [tokens, top_k], FP32
 *                accumulation, the coverage error, row and score gradients.
 *   [DS-AutoEP]  DeepSpeed AutoEP base PR, sections Attribution and Design:
 *                reorder tokens by expert, token-group alignment / padding for
 *                grouped GEMM, restore the original order.
 *   [DS-8190]    DeepSpeed PR "Derive AutoEP rank splits from the per-expert
 *                count exchange", sections Redundancy and Fix: the count
 *                matrix [ep_size, E_local], input_splits and
 *                received_counts.sum(dim=1) == output_splits.
 *   [XTuner-2056] XTuner PR "Integrate MoonEP dispatcher for FSDP
 *                expert-parallel training", Design and review: no host
 *                synchronisation on the hot path (histc, not bincount).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every data pointer is caller-owned DEVICE memory of the current device.
 *    The library allocates nothing and never synchronises with the host;
 *    every call only enqueues work on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream) and returns: kernels, plus for the folded
 *    restore's scatter one memset of its output.
 *    Results are defined once the stream reaches them.  The kernels use
 *    programmatic dependent launch: each waits for the kernel before it on
 *    the stream to complete before its first memory access, so the order the
 *    caller sees is plain stream order.  The only state kept between calls
 *    is per-device caches of launch attributes (SM count, shared-memory
 *    opt-ins) and the device array of moe_dispatch_layout_noalloc.
 *  - Notation: T tokens, H hidden size (bf16 elements per row), E experts,
 *    K = top_k, R logical ranks, El = E/R, align = group alignment,
 *    A = T*K assignments, flat index f = t*K + k (token t, slot k),
 *    N_cap = rows of the caller's expert-grouped buffers.
 *    Logical rank s owns tokens [s*T/R, (s+1)*T/R) as a source and experts
 *    [r*El, (r+1)*El) as a destination.  All arrays are row-major, densely
 *    packed.  bf16 values are passed as their uint16 bit patterns.
 *  - Return value: a HOST-detected error, MOE_OK (0) or a negative
 *    MOE_ERR_* code; on error nothing is enqueued.
 *  - `status` is one DEVICE int32 the caller zeroes before the first call;
 *    kernels OR MOE_ST_* bits into it when they meet bad data on the device.
 *    Outputs of a call that set a bit are undefined, but no kernel ever
 *    writes outside the buffers described here.  Read it after the stream
 *    has reached it (one synchronisation, when the caller chooses).
 *  - Limits: 1 <= K <= MOE_MAX_K, 1 <= E <= MOE_MAX_E, 1 <= R <= MOE_MAX_R,
 *    E % R == 0, T % R == 0, T >= 0, H > 0 and H % 8 == 0 (rows are whole
 *    16-byte vectors), A and N_cap < 2^31.  Row buffers must be 16-byte
 *    aligned, int64 arrays 8-byte, int32/float arrays 4-byte aligned.
 */
#ifndef MOE_DISPATCH_H
#define MOE_DISPATCH_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Host return codes. */
#define MOE_OK 0
#define MOE_ERR_INVALID_ARG (-1) /* a check listed under the call failed      */
#define MOE_ERR_CUDA (-2)        /* a CUDA runtime call or launch failed      */
#define MOE_ERR_SCRATCH (-3)     /* sizes need more than the static scratch of
                                    moe_dispatch_layout_noalloc              */

/* Device status bits (OR-ed into *status). */
#define MOE_ST_EXPERT_OOR 1       /* a topk_idx entry outside [0, E) (e.g. -1)  */
#define MOE_ST_CAPACITY 2         /* padded rows expert_offsets[E] > N_cap      */
#define MOE_ST_ROW_OOR 4          /* a flat_to_row entry outside [0, N_cap)     */
#define MOE_ST_COVERAGE 8         /* row maps do not cover each (token, slot) once */
#define MOE_ST_LAYOUT_MISMATCH 16 /* workspace was built for another (T, K, E)  */
#define MOE_ST_TIMEOUT 32         /* a bounded wait in a kernel gave up (outputs
                                     undefined; the kernel returned)         */

/* Routing-weight ("router") dtypes. */
#define MOE_DTYPE_F32 0
#define MOE_DTYPE_BF16 1

/* Bytes of the static device scratch behind moe_dispatch_layout_noalloc. */
#define MOE_NOALLOC_SCRATCH_BYTES (4u << 20)

#define MOE_MAX_K 32
#define MOE_MAX_E 1024
#define MOE_MAX_R 64

/* Bytes of the opaque layout workspace for (T, K, E, R).  The workspace is
 * written by moe_dispatch_layout and read by moe_permute (it plays the part of
 * the dispatch handle of [DeepEP-272]: per-tile expert bases and per-expert
 * counts).  Needs no initialisation.  Returns 0 for invalid sizes. */
size_t moe_layout_workspace_bytes(int T, int K, int E, int R);

/* A capacity that every routing fits: A + E*(align-1) rows (each expert
 * rounds its count up to a multiple of align).  Sizing the grouped buffers
 * with it removes the host wait for the actual count ([DeepEP-272],
 * num_worst_tokens).  Returns -1 for invalid sizes. */
int64_t moe_worst_case_rows(int T, int K, int E, int align);

/* Routing layout ([DeepEP-272] get_dispatch_layout; [DS-8190] count matrix;
 * [DS-AutoEP] group alignment).  Computed on the device only, with no host
 * synchronisation ([XTuner-2056]).
 *
 * In:  topk_idx [T,K] int64, entries in [0, E).
 * Out: tokens_per_expert [E] int32    c_e = #{f : topk_idx[f] = e}
 *      counts  [R,R,El] int32         counts[s][r][el] = assignments from
 *                                     source rank s to expert r*El+el (row s
 *                                     is rank s's count matrix [ep_size,
 *                                     E_local]; counts[:, r, :] is the
 *                                     received_counts of rank r)
 *      splits  [R,R] int32            splits[s][r] = sum_el counts[s][r][el]
 *                                     (row s = input_splits of rank s,
 *                                     column r = output_splits of rank r)
 *      tokens_per_rank [R,R] int32    distinct tokens of block s with some
 *                                     slot on rank r (num_tokens_per_rank)
 *      is_token_in_rank [T,R] uint8   1 iff some slot of t routes to rank r
 *      expert_offsets [E+1] int32     0, then running sum of
 *                                     ceil(c_e/align)*align (an empty expert
 *                                     takes no rows)
 *      workspace                      moe_layout_workspace_bytes(T,K,E,R)
 *                                     bytes, 16-byte aligned
 * Launch: two kernels, chained with programmatic dependent launch: one
 * 1024-thread CTA per tile of tokens ranks the assignments, then one warp per
 * row of per-tile counts scans it; the last of those CTAs writes the
 * offsets.  No memset, no grid barrier, no cooperative launch.
 * Status: MOE_ST_EXPERT_OOR (that assignment is left out of every count).
 * Errors: MOE_ERR_INVALID_ARG for a null pointer, sizes outside the limits,
 *         align < 1, misalignment. */
int moe_dispatch_layout(const int64_t* topk_idx, int T, int K, int E, int R, int align,
                        int32_t* tokens_per_expert, int32_t* counts, int32_t* splits,
                        int32_t* tokens_per_rank, uint8_t* is_token_in_rank,
                        int32_t* expert_offsets, void* workspace, int32_t* status,
                        cudaStream_t stream);

/* moe_dispatch_layout for callers that cannot allocate device memory.  The
 * pages have no counterpart of this call; it exists for callers such as a
 * plugin running inside a server or framework that owns the whole device
 * memory pool and only hands over the tensors it passes, or a path where
 * cudaMalloc/cudaFree must not run because they can synchronise the device.
 *
 * Same arguments, outputs, status bits and errors as moe_dispatch_layout,
 * minus `workspace`: the layout's scratch lives in one file-scope device
 * array of MOE_NOALLOC_SCRATCH_BYTES (4 MiB) that every GPU which loads the
 * library holds until the process exits.  The caller still passes all inputs
 * and outputs.  The call allocates nothing (no cudaMalloc, cudaFree or
 * allocating library routine).
 *  - Sizes whose workspace (moe_layout_workspace_bytes(T, K, E, R)) exceeds
 *    MOE_NOALLOC_SCRATCH_BYTES are rejected with MOE_ERR_SCRATCH and nothing
 *    is enqueued.
 *  - The first call on a device looks up the array's device address (with
 *    that device current) and caches it; make that first call before any
 *    stream capture on the device.  The cached address belongs to the
 *    device's context as it was at that first call: after cudaDeviceReset
 *    (which destroys that context and the library's device array with it)
 *    this call is not supported in the same process.
 *  - Every call shares the one array, which keeps the last call's contents;
 *    the call clears what must start at zero (its first kernel zeroes the
 *    arrival counter its second kernel counts on) and its kernels write every
 *    other word they read before reading it, so the caller clears nothing.
 *    Calls that overlap on the GPU -- on different streams, or from threads
 *    whose streams are not ordered -- race on it and give undefined results.
 *  - The permute cannot use this scratch; a caller that also permutes uses
 *    moe_dispatch_layout with its own workspace. */
int moe_dispatch_layout_noalloc(const int64_t* topk_idx, int T, int K, int E, int R, int align,
                                int32_t* tokens_per_expert, int32_t* counts, int32_t* splits,
                                int32_t* tokens_per_rank, uint8_t* is_token_in_rank,
                                int32_t* expert_offsets, int32_t* status, cudaStream_t stream);

/* Dispatch on one device ([DeepEP-272] dispatch; [DS-AutoEP] step 3,
 * "reorder tokens by expert assignment").  Assignment f = (t, k) with
 * e = topk_idx[f] is written to
 *
 *   row(f) = expert_offsets[e] + #{f' < f : topk_idx[f'] = e}
 *
 * (stable order: expert, then token, then slot):
 *   x_perm[row(f)] = x[t],  flat_to_row[f] = row(f),  row_to_flat[row(f)] = f.
 * Pad rows [off[e] + c_e, off[e+1]) get row_to_flat = -1 and, when zero_pad
 * is non-zero, zero contents.  Rows [off[E], N_cap) get row_to_flat = -1 and
 * keep their contents.
 *
 * In:  x [T,H] bf16; topk_idx [T,K] int64; expert_offsets and workspace from
 *      moe_dispatch_layout with the same (topk_idx, T, K, E).
 * Out: x_perm [N_cap,H] bf16, row_to_flat [N_cap] int32, flat_to_row [T,K]
 *      int32 (-1 for an assignment that was not placed).
 * Status: MOE_ST_CAPACITY (rows >= N_cap are not written),
 *         MOE_ST_EXPERT_OOR, MOE_ST_LAYOUT_MISMATCH (nothing written),
 *         MOE_ST_TIMEOUT (K <= 2: a bounded wait on the kernel's own
 *         shared-memory copies gave up; outputs undefined).
 * Errors: MOE_ERR_INVALID_ARG as for the layout, or N_cap < A. */
int moe_permute(const uint16_t* x, const int64_t* topk_idx, int T, int K, int E, int H,
                const int32_t* expert_offsets, const void* workspace, int zero_pad,
                int64_t N_cap, uint16_t* x_perm, int32_t* row_to_flat, int32_t* flat_to_row,
                int32_t* status, cudaStream_t stream);

/* The layout and the permute in one call ([DeepEP-272]: the layout, then
 * the dispatch with its handle): moe_dispatch_layout, then moe_permute on its
 * outputs, with the arguments, outputs, status bits and errors of both; every
 * check of both runs before anything is enqueued, so an invalid argument
 * leaves the stream untouched.  The workspace is filled as by
 * moe_dispatch_layout and may be passed on to moe_permute_payload and the
 * other calls that take a layout. */
int moe_dispatch(const uint16_t* x, const int64_t* topk_idx, int T, int K, int E, int R, int H,
                 int align, int32_t* tokens_per_expert, int32_t* counts, int32_t* splits,
                 int32_t* tokens_per_rank, uint8_t* is_token_in_rank, int32_t* expert_offsets,
                 void* workspace, int zero_pad, int64_t N_cap, uint16_t* x_perm,
                 int32_t* row_to_flat, int32_t* flat_to_row, int32_t* status,
                 cudaStream_t stream);

/* Stand-in expert between dispatch and combine: for each expert e, its real
 * rows [off[e], off[e] + c_e) become bf16_rn(fp32(row) * scales[e]) (the
 * product rounded to fp32, then once to bf16); its pad rows become zero;
 * rows >= off[E] are untouched.  In the backward pass the same call maps row
 * gradients to input-row gradients (d(x*s)/dx = s).  It stands where the
 * grouped expert MLP of [DS-AutoEP] (Design, step 5) runs.
 *
 * In:  rows [N_cap,H] bf16; expert_offsets [E+1]; tokens_per_expert [E];
 *      scales [E] fp32.   Out: out [N_cap,H] bf16 (may not alias rows).
 * Status: MOE_ST_CAPACITY if off[E] > N_cap (nothing past N_cap is touched). */
int moe_expert_scale(const uint16_t* rows, int64_t N_cap, const int32_t* expert_offsets,
                     const int32_t* tokens_per_expert, int E, int H, const float* scales,
                     uint16_t* out, int32_t* status, cudaStream_t stream);

/* fused_weighted_restore ([DS-8847] Change; [DeepEP-272] combine):
 *
 *   acc = 0;  for k = 0..K-1:  acc = fmaf(w[t,k], rows[flat_to_row[t*K+k]], acc)
 *   out[t] = bf16_rn(acc)
 *
 * per element, FP32, fixed slot order, one rounding.  weights [T,K] are in the
 * router dtype (weight_dtype = MOE_DTYPE_F32 or MOE_DTYPE_BF16, widened
 * exactly); weights = NULL means unit weights, which is the backward of
 * dispatch ([DeepEP-272]: "the backward process of MoE dispatch is actually a
 * combine").  A slot whose row is outside [0, N_cap) contributes nothing and
 * sets MOE_ST_ROW_OOR.
 *
 * validate != 0 adds the coverage check of [DS-8847] ("raises a clear
 * RuntimeError if the gathered rows do not cover every (token, slot)"):
 * row_to_flat[flat_to_row[f]] == f for every f, and
 * flat_to_row[row_to_flat[r]] == r for every row with row_to_flat[r] >= 0;
 * a failure sets MOE_ST_COVERAGE.  row_to_flat may be NULL when validate == 0.
 *
 * In:  rows [N_cap,H] bf16, maps from moe_permute.   Out: out [T,H] bf16. */
int moe_combine_weighted(const uint16_t* rows, int64_t N_cap, const int32_t* row_to_flat,
                         const int32_t* flat_to_row, const void* weights, int weight_dtype,
                         int T, int K, int H, int validate, uint16_t* out, int32_t* status,
                         cudaStream_t stream);

/* ------------------------------------------------ payload and fp32 rows ---
 * [DeepEP-272]: dispatch takes x either as a bf16 tensor or as an FP8 tuple
 * (data, scales); [DS-8847] Tests: the fused restore on "fp32 and bf16 rows". */

/* Dispatch of an opaque row payload: exactly moe_permute (same rows, maps,
 * pad rows, tail, status bits and layout workspace) for rows of any byte
 * width, plus an optional per-token aux row that goes to the same rows.
 *
 *   x_perm[row(f)] = x[t]         aux_perm[row(f)] = aux[t]
 *
 * FP8 tuple: x = e4m3 data [T,H] (row_bytes = H), aux = fp32 scales
 * [T, H/128] (aux_row_bytes = 4*H/128).  fp32 rows: row_bytes = 4*H, aux NULL.
 * In:  x [T, row_bytes] (16-byte aligned, row_bytes a positive multiple of
 *      16); aux [T, aux_row_bytes] (4-byte aligned; aux_row_bytes a multiple
 *      of 4, at most 65536; 0 means no aux payload and both aux pointers are
 *      ignored).
 * Out: x_perm [N_cap, row_bytes]; aux_perm [N_cap, aux_row_bytes];
 *      row_to_flat [N_cap]; flat_to_row [T,K].  With zero_pad, pad rows of
 *      both payloads are zero.  aux may be NULL only when T == 0 and
 *      aux_perm only when N_cap == 0.
 * Errors: MOE_ERR_INVALID_ARG as for moe_permute, or a row width outside
 *         the rules above. */
int moe_permute_payload(const void* x, int64_t row_bytes, const void* aux, int64_t aux_row_bytes,
                        const int64_t* topk_idx, int T, int K, int E,
                        const int32_t* expert_offsets, const void* workspace, int zero_pad,
                        int64_t N_cap, void* x_perm, void* aux_perm, int32_t* row_to_flat,
                        int32_t* flat_to_row, int32_t* status, cudaStream_t stream);

/* fused_weighted_restore on fp32 rows: moe_combine_weighted with rows and
 * out in fp32 (the activation dtype), the same FP32 fmaf chain in slot order
 * and no final rounding:
 *
 *   out[t] = fmaf chain over k of (w[t,k], rows[flat_to_row[t*K+k]])
 *
 * Weights, validation and status exactly as moe_combine_weighted; H % 4 == 0
 * (16-byte rows); rows and out 16-byte aligned. */
int moe_combine_weighted_f32(const float* rows, int64_t N_cap, const int32_t* row_to_flat,
                             const int32_t* flat_to_row, const void* weights, int weight_dtype,
                             int T, int K, int H, int validate, float* out, int32_t* status,
                             cudaStream_t stream);

/* Backward of the fp32-row restore: moe_combine_backward with grad_out, rows
 * and grad_rows in fp32:
 *
 *   grad_rows[flat_to_row[f]] = fp32(w[f] * g[t])      (one rounding)
 *   grad_weights[f] = sum_h g[t,h] * rows[flat_to_row[f], h]
 *
 * fp32 x fp32 products are exact in fp64 and summed in fp64, then rounded
 * once to the router dtype.  Everything else as moe_combine_backward. */
int moe_combine_backward_f32(const float* grad_out, const float* rows, int64_t N_cap,
                             const int32_t* row_to_flat, const int32_t* flat_to_row,
                             const void* weights, int weight_dtype, int T, int K, int H,
                             const int32_t* expert_offsets, int E, int zero_pad,
                             float* grad_rows, void* grad_weights, int32_t* status,
                             cudaStream_t stream);

/* Scatter step of the folded restore ([DS-8847] Change: the rows of all
 * tensor-parallel peers are gathered together with ONE flat index per row,
 * token * top_k + slot; the routing data is scattered into [tokens, top_k];
 * a clear RuntimeError is raised if the gathered rows do not cover every
 * (token, slot)).  Builds the map moe_combine_weighted needs from the
 * gathered rows' flat indices:
 *
 *   flat_to_row[f] = the row r with row_flat[r] == f
 *
 * In:  row_flat [N] int32 -- the flat index each gathered row holds, -1 for a
 *      row holding none (a pad row).
 * Out: flat_to_row [T,K] int32.
 * Status: MOE_ST_COVERAGE if some f in [0, T*K) is held by no row or by more
 *         than one, or a row holds an index outside [-1, T*K); flat_to_row is
 *         then undefined.  Enqueues a memset and two small kernels. */
int moe_scatter_flat_index(const int32_t* row_flat, int64_t N, int T, int K,
                           int32_t* flat_to_row, int32_t* status, cudaStream_t stream);

/* Row labels from segment counts: the receive side of expert parallelism
 * across GPUs ([DS-8190] Redundancy: received_counts[s, e] is the number of
 * rows source rank s sends to local expert e; after the payload all-to-all
 * they arrive source by source, each source's rows in local-expert order).
 * Row i of a buffer of n consecutive segments, segment j holding counts[j]
 * rows, gets
 *
 *   labels[i] = j % modulo        (received buffer: j = s*E_local + e,
 *                                  modulo = E_local, label = local expert)
 *
 * and rows past sum(counts) get -1.  The labels, read as topk_idx [rows, 1],
 * let moe_dispatch_layout + moe_permute regroup the received rows by local
 * expert (stable: source rank, then the source's order).
 * In:  counts [n] int32 (device), 1 <= n <= MOE_MAX_E, modulo >= 1,
 *      0 <= rows <= INT32_MAX.
 * Out: labels [rows] int64 (device, 8-byte aligned).
 * Status: MOE_ST_CAPACITY if sum(counts) > rows (the rows past `rows` are not
 *         labelled), MOE_ST_COVERAGE if a count is negative (counted as 0).
 * Errors: MOE_ERR_INVALID_ARG for sizes outside the limits, a null pointer or
 *         misalignment.  One kernel. */
int moe_segment_labels(const int32_t* counts, int n, int modulo, int64_t rows, int64_t* labels,
                       int32_t* status, cudaStream_t stream);

/* Row bases of expert parallelism without a send buffer ([DS-8190]
 * Redundancy and Fix: every rank derives where its rows go from the
 * per-expert counts of all ranks, exchanged once; [DS-AutoEP] Attribution:
 * group alignment).  The receive buffer of owner rank r holds its experts
 * [r*El, (r+1)*El) in order, each group padded to a multiple of align, and
 * inside a group the rows of source rank 0, then 1, ...  From all_counts
 * [R,E] int32 (row s = tokens_per_expert of source rank s's own tokens):
 *
 *   dest_base[e]     = start of e's group in its owner's buffer
 *                      + sum over s < rank of all_counts[s][e]
 *   own_offsets[el]  = start of group el in rank `rank`'s own buffer,
 *   own_offsets[El]  = that buffer's padded total
 *   own_counts[el]   = sum over s of all_counts[s][rank*El + el]
 *   max_rows[0]      = the largest padded total over the R owners (the rows
 *                      every receive buffer needs for this routing)
 *
 * The inputs of moe_permute_to_ranks (dest_base, own_offsets, own_counts);
 * computed on the device, so the only host copy of the plan is the caller's
 * read of max_rows when it sizes the buffers.
 * In:  all_counts [R,E] int32 (device).
 * Out: dest_base [E], own_offsets [E/R + 1], own_counts [E/R], max_rows [1]
 *      int32 (device).
 * Status: MOE_ST_COVERAGE for a negative count (counted as 0),
 *         MOE_ST_CAPACITY if a padded group would overflow int32.
 * Errors: MOE_ERR_INVALID_ARG for R outside [1, MOE_MAX_R], E outside
 *         [1, MOE_MAX_E], E % R, rank outside [0, R), align < 1, a null
 *         pointer or misalignment.  One kernel of one CTA. */
int moe_rank_bases(const int32_t* all_counts, int R, int E, int rank, int align,
                   int32_t* dest_base, int32_t* own_offsets, int32_t* own_counts,
                   int32_t* max_rows, int32_t* status, cudaStream_t stream);

/* Dispatch straight into the receive buffers of the ranks that own the
 * experts (expert parallelism across GPUs without a send buffer; [DeepEP-272]
 * dispatch sends token rows to the ranks owning their experts; [DS-8190] the
 * per-(source rank, expert) counts the offsets come from).  Rank `rank` of R,
 * holding T tokens, stores assignment f = (t, k) of expert e into the buffer
 * of rank r = e / (E/R) at
 *
 *   row(f) = dest_base[e] + #{f' < f of this rank's tokens : topk_idx[f'] = e}
 *
 * where dest_base[e] = (start of e's padded group in rank r's buffer) + (rows
 * of e sent by ranks before `rank`), so every receive buffer comes out in the
 * order the single-device layout gives those experts (source rank, token,
 * slot), padded per expert to the group alignment.  The pad rows of this
 * rank's OWN receive buffer are zeroed here when zero_pad != 0 (every rank
 * zeroes its own).
 * In:  x [T,H] bf16, topk_idx [T,K] int64, dest_base [E] int32 (device),
 *      workspace: moe_dispatch_layout of these T tokens with R = 1 (its
 *      in-tile ranks; checked on the device: MOE_ST_LAYOUT_MISMATCH),
 *      dest_rows: DEVICE array of R pointers to bf16 buffers [dest_cap, H]
 *      (16-byte aligned; across GPUs, peer addresses of the other ranks'
 *      buffers, written with plain stores), dest_claims: NULL, or a DEVICE
 *      array of R pointers to int32 arrays [dest_cap] beside those buffers:
 *      every row stored gets the claim (rank << 25) | f, and this rank's own
 *      pad rows and rows past its padded total get -1 (needs T*K <= 2^25),
 *      own_offsets [E/R + 1] and own_counts [E/R] int32: this rank's padded
 *      group starts and real rows.
 * Out: the rows in the ranks' buffers; flat_to_row [T,K] int32 = row(f) in
 *      the buffer of its expert's rank (-1 if none).
 * Status: MOE_ST_EXPERT_OOR, MOE_ST_CAPACITY (a row at or past dest_cap is
 *         not written), MOE_ST_LAYOUT_MISMATCH.
 * Errors: MOE_ERR_INVALID_ARG for sizes outside the limits (also E % R,
 *         rank outside [0, R)), a null pointer or misalignment.  The caller
 *         orders the ranks' calls before any reader of the buffers (across
 *         GPUs: a barrier between this call and the experts). */
int moe_permute_to_ranks(const uint16_t* x, const int64_t* topk_idx, int T, int K, int E, int R,
                         int H, const int32_t* dest_base, const void* workspace,
                         uint16_t* const* dest_rows, int32_t* const* dest_claims,
                         int64_t dest_cap, int rank, const int32_t* own_offsets,
                         const int32_t* own_counts, int zero_pad, int32_t* flat_to_row,
                         int32_t* status, cudaStream_t stream);

/* Combine straight out of the ranks' expert-output buffers: the
 * fused_weighted_restore of [DS-8847] for this rank's T tokens, slot (t, k)
 * read from the buffer of rank topk_idx[t,k] / (E/R) at row flat_to_row[t,k]
 * (as moe_permute_to_ranks wrote it):
 *
 *   out[t] = bf16_rn(fmaf chain over k of w[t,k] * rows[rank][flat_to_row[t,k]])
 *
 * the same FP32 slot-order chain as moe_combine_weighted, so the result is
 * bit-identical to the single-device restore of the same rows.
 * In:  rows: DEVICE array of R pointers to bf16 [N_cap, H] buffers (across
 *      GPUs, peer addresses; plain loads), flat_to_row [T,K], topk_idx [T,K],
 *      weights [T,K] fp32 or bf16; claims: NULL, or the DEVICE array of R
 *      claim arrays that moe_permute_to_ranks filled (peer addresses across
 *      GPUs), with `rank` this rank's index.
 * Out: out [T,H] bf16.
 * Status: MOE_ST_ROW_OOR for a slot whose row or expert is out of range (it
 *         contributes nothing).  With claims, the coverage check of [DS-8847]
 *         from the slot side: every slot's row must be claimed by exactly this
 *         (rank, token, slot), else MOE_ST_COVERAGE -- a duplicated, stale or
 *         foreign row is caught.  (Rows nobody points to are not visible to
 *         one rank.)
 * Errors: MOE_ERR_INVALID_ARG as moe_combine_weighted, plus E % R, and with
 *         claims rank outside [0, R) or T*K > 2^25. */
int moe_combine_from_ranks(const uint16_t* const* rows, const int32_t* const* claims, int R,
                           int rank, int64_t N_cap, const int32_t* flat_to_row,
                           const int64_t* topk_idx, int E, const void* weights, int weight_dtype,
                           int T, int K, int H, uint16_t* out, int32_t* status,
                           cudaStream_t stream);

/* Backward of fused_weighted_restore ([DS-8847] Tests: row and score
 * gradients; Benchmark: score gradient in FP32; [DeepEP-272]: the backward
 * of combine is a dispatch).  With g = grad_out [T,H]:
 *
 *   grad_rows[flat_to_row[f]] = bf16_rn(fp32(w[f] * g[t]))
 *   grad_weights[f] = sum_h g[t,h] * rows[flat_to_row[f], h]
 *
 * grad_weights: bf16 x bf16 products are exact in fp32 and are summed in
 * fp64, then rounded once to the router dtype; it may be NULL.  When zero_pad
 * is non-zero, every row below expert_offsets[E] whose row_to_flat is
 * negative (a pad row) is written as zero; rows >= off[E] are untouched.
 * row_to_flat may be NULL when zero_pad == 0.
 *
 * In:  grad_out [T,H] bf16; rows [N_cap,H] bf16 (the forward's combine input);
 *      maps; weights [T,K] (router dtype, not NULL); expert_offsets [E+1].
 * Out: grad_rows [N_cap,H] bf16; grad_weights [T,K] router dtype.
 * Status: MOE_ST_ROW_OOR (that slot is skipped and its weight gradient is 0). */
int moe_combine_backward(const uint16_t* grad_out, const uint16_t* rows, int64_t N_cap,
                         const int32_t* row_to_flat, const int32_t* flat_to_row,
                         const void* weights, int weight_dtype, int T, int K, int H,
                         const int32_t* expert_offsets, int E, int zero_pad,
                         uint16_t* grad_rows, void* grad_weights, int32_t* status,
                         cudaStream_t stream);

/* Static text for a return code (MOE_OK / MOE_ERR_*) or for ONE status bit. */
const char* moe_strerror(int code);
const char* moe_status_bit_name(int bit);

/* The name of the CUDA error (e.g. "cudaErrorIllegalAddress") behind the
 * calling host thread's most recent MOE_ERR_CUDA return, or "none".  Static
 * text; a later MOE_ERR_CUDA on the same thread replaces it.  A sticky
 * error from an earlier kernel surfaces at the next launch, so the call
 * that reports it need not be the one whose kernel failed. */
const char* moe_last_cuda_error(void);

/* Library version string. */
const char* moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_DISPATCH_H */

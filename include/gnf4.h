/*
 * gnf4.h -- C ABI of libgnf4: the grouped Mixture-of-Experts expert GEMM
 * computed directly on 4-bit-packed weights, on one NVIDIA B200 (sm_100a).
 *
 * The operation (grouped-nf4-gemm 0.33.1 on PyPI, opening paragraphs): one
 * launch runs the expert GEMM for every routed expert, decoding the packed
 * weights in registers with their block scale, accumulating in fp32 and
 * writing bf16.  No bf16 copy of any expert is ever written to memory.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All array pointers are DEVICE pointers, allocated and owned by the
 *    caller.  libgnf4 allocates nothing, frees nothing and keeps no pointer
 *    after a call returns.  A host pointer is refused (GNF4_ERR_INVALID_ARG)
 *    before any launch: nothing ever falls back to the CPU (grouped-nf4-gemm
 *    index.json, "non_goals": no silent fallbacks).
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Calls only enqueue work on it; none synchronises the host.
 *  - Inputs are never written (grouped-nf4-gemm releases, v0.2.5 "Fix:
 *    build_group_tiles mutated its sizes argument").
 *  - Shapes and alignment are checked on the host before launch and refused
 *    with GNF4_ERR_UNSUPPORTED_SHAPE (grouped-nf4-gemm status page, "#324's
 *    pre-launch shape refusal").  Byte offsets into the expert stacks are
 *    64-bit (same page, "#87 ... int32 offset overflow").
 *  - Errors that only the device can see (offsets that are not monotone or
 *    exceed M, a GEMV group with more than 8 rows, a pipeline wait that ran
 *    out) set bits in a device-side error word; read it with
 *    gnf4_device_errors().
 *  - gnf4_last_error() returns the text of the calling thread's last failure.
 *
 * Layouts
 * -------
 *  bf16 activations A / x / y / out are row-major, rows contiguous.
 *  NF4 stack (bitsandbytes gemm_4bit layout; grouped-nf4-gemm 0.33.1 on
 *    PyPI, "Try it on CPU right now", example 1):
 *      w      uint8 [E, N, K/2]  two codes per byte, element 2i in the HIGH
 *                                nibble, element 2i+1 in the LOW nibble;
 *      absmax fp32  [E, N, K/64] one scale per 64 consecutive elements of a
 *                                row; value = NF4[code] * absmax.
 *  MXFP4 stack (OCP e2m1 + e8m0; same page, example 2, and grouped-nf4-gemm
 *    releases, v0.2.5 "arena -> kernel"):
 *      w      uint8 [E, N, K/2]  element 2i in the LOW nibble, 2i+1 in the
 *                                HIGH nibble; bit 3 of a nibble is the sign;
 *      scales uint8 [E, N, K/32] e8m0: value = e2m1[code] * 2^(scale-127).
 *  Group description: `offsets` int32 [E+1] (rows of expert e are
 *    offsets[e] .. offsets[e+1]-1 of the group-sorted A and Y, offsets[0] = 0,
 *    offsets[E] <= M) or `counts` int32 [E] (per-group row count, the
 *    pages' `sizes`: grouped-nf4-gemm releases, v0.3.1 "sizes is a per-group
 *    token count").  Exactly one of the two is non-NULL.
 *  Y[r, n] = sum_k A[r, k] * W_e[n, k] for offsets[e] <= r < offsets[e+1]
 *    (both operands K-major).  Rows r >= offsets[E] of Y are not written.
 */
#ifndef GNF4_H
#define GNF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GNF4_OK = 0,
    GNF4_ERR_INVALID_ARG = 1,       /* NULL / host / misaligned pointer, bad count */
    GNF4_ERR_UNSUPPORTED_SHAPE = 2, /* a shape rule below is broken */
    GNF4_ERR_CUDA = 3,              /* a CUDA runtime call or launch failed */
    GNF4_ERR_TIMEOUT = 4            /* reported through gnf4_device_errors() */
} gnf4_status;

/* Bits of the device error word (gnf4_device_errors). */
#define GNF4_DEVERR_TIMEOUT 0x1u      /* a bounded pipeline wait gave up; outputs incomplete */
#define GNF4_DEVERR_BAD_OFFSETS 0x2u  /* offsets not monotone, offsets[0] != 0 or offsets[E] > M */
#define GNF4_DEVERR_GEMV_ROWS 0x4u    /* a GEMV group held more than 8 rows; that group was skipped */
#define GNF4_DEVERR_INTERNAL 0x8u     /* a kernel's shared-memory layout check failed; no output written */

/* Text of the calling thread's last failure ("" if none). */
const char *gnf4_last_error(void);

/* Library version string. */
const char *gnf4_version(void);

/* Reads (and if `clear` != 0, resets) the device error word of the current
 * device into *flags.  Synchronises the device: diagnostics only, never on
 * the hot path. */
gnf4_status gnf4_device_errors(uint32_t *flags, int clear);

/* Failure-detection self-test: enqueues one kernel whose single thread runs
 * the pipelines' bounded mbarrier wait on a barrier that nothing ever
 * arrives on, giving up after limit_cycles SM clock cycles (1 .. 2^32).  On
 * return of the kernel the device error word holds GNF4_DEVERR_TIMEOUT and
 * the context stays usable.  No fault, trap or unbounded spin is involved. */
gnf4_status gnf4_selftest_bounded_wait(unsigned long long limit_cycles, void *stream);

/* ------------------------------------------------------------------ */
/* Engagement counters                                                  */
/* ------------------------------------------------------------------ */

/* A returned status says that a call was accepted; these counters say
 * whether it reached a kernel, and which kernel family ran (grouped-nf4-gemm
 * releases, v0.2.6 "Honest instrumentation": a patch count is not a call
 * count; status page, "What is open": a silent fallback made countable).
 * One record per entry point that enqueues work, kept on the host,
 * process-wide (all devices, all threads), updated with relaxed atomics;
 * counting needs no device and no synchronisation.  A call that another
 * entry point makes on the caller's behalf (gnf4_route_permute_static runs
 * gnf4_route_permute) counts under the outer entry point only.
 *
 * Which kernels a call launches is decided on the host; which groups a
 * launched kernel then finds work in is decided on the device from the
 * offsets (gnf4_grouped_gemm_mxfp4_ws launches the native kernel for groups
 * of at most gnf4_grouped_gemm_mxfp4_native_max_rows() rows and, when
 * M exceeds that, the decode-path kernel for the larger ones). */
typedef struct {
    uint64_t calls;       /* times the entry point was called */
    uint64_t refused;     /* calls that returned a status other than GNF4_OK */
    uint64_t engaged;     /* calls that enqueued work (a kernel, or a memset) */
    uint64_t rows;        /* summed over engaged calls: M for the grouped
                             and quantiser calls, T*k for routing and the
                             separate combine, weight rows for dequant */
    uint64_t decode_path; /* engaged calls that launched a tensor-core kernel
                             on decoded weights (kind::f16: GEMM, SwiGLU
                             GEMM, fused-combine GEMM, dgrad) */
    uint64_t native_path; /* engaged calls that launched the native
                             block-scaled kernel (W4A8, two-term, W4A4) */
    uint64_t gemv_path;   /* engaged calls that launched the decode GEMV */
} gnf4_call_stats;

/* Copies the counters of the entry point named `entry` (its C name, e.g.
 * "gnf4_grouped_gemm_mxfp4_ws") into *out, or their sums over every entry
 * point when `entry` is NULL; with `reset` != 0 those counters are then set
 * to zero.  GNF4_ERR_INVALID_ARG for a NULL `out` or a name that is not
 * counted (nothing is reset then). */
gnf4_status gnf4_call_stats_get(const char *entry, gnf4_call_stats *out, int reset);

/* Name of the i-th counted entry point (0-based), or NULL past the last. */
const char *gnf4_call_stats_name(int i);

/* ------------------------------------------------------------------ */
/* Routing: sort (token, slot) pairs into per-expert row groups         */
/* ------------------------------------------------------------------ */

/* Workspace bytes gnf4_route_permute needs for T tokens, top-k, E experts. */
size_t gnf4_route_workspace_bytes(int T, int k, int E);

/* Stable counting sort of the M = T*k (token, slot) pairs by expert id and
 * gather of the activations into group-sorted order (grouped-nf4-gemm
 * releases, v0.2.6 "The patch point": argsort of the top-k ids, the gather
 * x[idxs // k], and tokens_per_expert as the group sizes).
 *   topk_ids       int32 [T, k]   expert of pair f = t*k + j;
 *   x              bf16  [T, K]   token activations;
 *   offsets        int32 [E+1]    OUT: group row offsets, offsets[E] = valid pairs;
 *   sorted_to_flat int32 [M]      OUT: pair of each sorted row, -1 past offsets[E];
 *   flat_to_sorted int32 [M]      OUT: sorted row of each pair, -1 if dropped;
 *   x_sorted       bf16  [M, K]   OUT: x_sorted[r] = x[sorted_to_flat[r] / k];
 *                                 rows past offsets[E] are zero;
 *   workspace      device bytes, at least gnf4_route_workspace_bytes(T, k, E),
 *                  16-byte aligned; its contents on entry do not matter;
 *   bad_id_count   int32 [1] OUT (may be NULL): pairs whose id is outside
 *                  [0, E).  Such pairs are dropped, never used as an index
 *                  (grouped-nf4-gemm releases, v0.3.0 "Also": model-global
 *                  expert ids read out of bounds silently).
 * Within an expert, pairs keep ascending flat index (a stable sort).
 * Rules: T >= 0, 1 <= k <= E <= 4096, T*k <= 2^30, K >= 8 and K % 8 == 0,
 * x and x_sorted 16-byte aligned.  T == 0 writes offsets only. */
gnf4_status gnf4_route_permute(const int32_t *topk_ids, const void *x, int T, int k, int E, int K,
                               int32_t *offsets, int32_t *sorted_to_flat, int32_t *flat_to_sorted,
                               void *x_sorted, void *workspace, size_t workspace_bytes,
                               int32_t *bad_id_count, void *stream);

/* Allocation-free variant of gnf4_route_permute.  The pages have no
 * counterpart to this call; it exists for callers that cannot allocate
 * device memory -- e.g. a plugin inside an inference engine whose device
 * memory is budgeted and owned by the host process, or latency-critical code
 * that must not pay for cudaMalloc's implicit synchronisation.  It computes
 * exactly what gnf4_route_permute computes, with the same arguments minus
 * the workspace: its scratch is a fixed array of
 * GNF4_ROUTE_STATIC_SCRATCH_BYTES bytes compiled into the library, one copy
 * on every GPU that loads libgnf4, held until the process exits.
 *  - Shapes whose scratch (gnf4_route_workspace_bytes(T, k, E)) exceeds the
 *    array are refused with GNF4_ERR_UNSUPPORTED_SHAPE; use
 *    gnf4_route_permute with your own workspace for those.
 *  - The first call on a device looks up the array's device address (once
 *    per device, with that device current); make that first call before any
 *    stream capture begins.
 *  - Every call on a device shares the one array and leaves its contents
 *    behind; nothing in it needs to start at zero.  Calls whose executions
 *    overlap on the GPU (different streams, no ordering between them) race
 *    on the array: order them.
 *  - It never calls cudaMalloc, cudaFree or any allocating routine. */
#define GNF4_ROUTE_STATIC_SCRATCH_BYTES ((size_t)1 << 20)
gnf4_status gnf4_route_permute_static(const int32_t *topk_ids, const void *x, int T, int k, int E, int K,
                                      int32_t *offsets, int32_t *sorted_to_flat, int32_t *flat_to_sorted,
                                      void *x_sorted, int32_t *bad_id_count, void *stream);

/* ------------------------------------------------------------------ */
/* Router epilogue + routing                                           */
/* ------------------------------------------------------------------ */

/* The router's softmax and top-k fused with the routing above
 * (grouped-nf4-gemm index.json, problems_solved[5]: router softmax and
 * top-k among the decode tail folded into one launch; entrypoints:
 * int4_b32:router_epilogue).  For every token t, with score[e] =
 * logits[t, e] + bias[e] computed in fp32 (bias NULL = no bias):
 *   topk_ids[t, 0..k)     the k distinct experts with the largest scores,
 *                         descending; ties go to the lower expert index;
 *                         NaN scores rank below every number;
 *   topk_weights[t, j]    softmax over the k selected RAW logits (the bias
 *                         moves the selection only), fp32;
 * then offsets, sorted_to_flat, flat_to_sorted and x_sorted exactly as
 * gnf4_route_permute computes them from topk_ids.
 *
 * logits: device fp32 [T, E] (4-byte aligned); bias: device fp32 [E] or
 * NULL; x: bf16 [T, K]; outputs as gnf4_route_permute plus topk_ids int32
 * [T, k] and topk_weights fp32 [T, k].  1 <= k <= min(E, 32), E <= 4096,
 * other shape rules as gnf4_route_permute; workspace as
 * gnf4_route_workspace_bytes(T, k, E).  T*k <= 256 runs as one
 * launch.  The pages fix no tie rule or weight convention: this is a
 * reading. */
gnf4_status gnf4_route_topk_permute(const float *logits, const float *bias, int T, int E, int k, const void *x, int K,
                                    int32_t *topk_ids, float *topk_weights, int32_t *offsets,
                                    int32_t *sorted_to_flat, int32_t *flat_to_sorted, void *x_sorted,
                                    void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------ */
/* Grouped GEMM (prefill: any number of rows per group)                */
/* ------------------------------------------------------------------ */

/* NF4 grouped GEMM on tcgen05 tensor cores (grouped-nf4-gemm 0.33.1 on PyPI,
 * opening paragraphs; grouped-nf4-gemm index.json, problems_solved[0]).
 *   a      bf16 [M, K] group-sorted activations (16-byte aligned);
 *   w, absmax: the NF4 stack above (w 16-byte aligned);
 *   offsets / counts: the group description above;
 *   y      bf16 [M, N] OUT.
 * Rules: 1 <= E <= 1024, N >= 1, N % 8 == 0, K % 64 == 0, 64 <= K <= 65536,
 * M >= 0 (M == 0 launches nothing).  Decoded weights are rounded to bf16 for
 * the tensor-core multiply; sums are fp32; the output is rounded to bf16. */
gnf4_status gnf4_grouped_gemm_nf4(const void *a, const uint8_t *w, const float *absmax, const int32_t *offsets,
                                  const int32_t *counts, int E, int N, int K, int M, void *y, void *stream);

/* MXFP4 grouped GEMM (grouped-nf4-gemm releases, v0.2.0 "the MXFP4
 * native-byte lane": the e2m1 codebook is a table swap of the NF4 mainloop;
 * v0.3.1: gemm_mxfp4_grouped's sizes is a per-group token count).
 * Same arguments with `scales` (e8m0 [E, N, K/32]) for absmax.
 * Rules: as NF4 but K % 32 == 0, 32 <= K <= 65536.  e2m1 times a power of two
 * is exact in bf16, so the tensor cores see the exact decoded weights. */
gnf4_status gnf4_grouped_gemm_mxfp4(const void *a, const uint8_t *w, const uint8_t *scales, const int32_t *offsets,
                                    const int32_t *counts, int E, int N, int K, int M, void *y, void *stream);

/* The same MXFP4 grouped GEMM with the native block-scaled path for small
 * groups (grouped-nf4-gemm releases, v0.2.0 "the MXFP4 native-byte lane";
 * bw24 v0.9.0, Documentation "prefill arc design": the e2m1 stack read as it
 * is by a block-scaled MMA).  Same arguments, rules and result tolerance as
 * gnf4_grouped_gemm_mxfp4, plus a caller-owned device workspace:
 *   - groups of at most gnf4_grouped_gemm_mxfp4_native_max_rows() (96) rows:
 *     their activation rows are split into two MXFP8 terms in the workspace
 *     (the rule of gnf4_quantize_mxfp8_split) and multiplied on tcgen05
 *     kind::mxf8f6f4 against the stack unchanged, nothing decoded on the SM;
 *   - larger groups: the decode path of gnf4_grouped_gemm_mxfp4.
 * On B200 the native path takes about half the time of the decode path per
 * group of up to 96 rows; a larger group needs one native unit per 96 rows
 * per weight tile, which the decode path covers with one per 256.
 *
 * workspace: NULL (every group takes the decode path, nothing else is
 * needed), or device memory of at least
 * gnf4_grouped_gemm_mxfp4_workspace_bytes(M, K) bytes, 16-byte aligned; a
 * smaller non-NULL workspace is refused with GNF4_ERR_INVALID_ARG.  Its
 * contents are scratch: written and read within the call's stream order.
 * When K % 64 != 0 or K < 128 the native path does not apply: the workspace
 * size is 0 and every group takes the decode path; so does every group when
 * E*N >= 2^31.  With a workspace, w must
 * be 32-byte aligned.  Up to three launches (split quantiser, native GEMM,
 * decode GEMM; the last is skipped when M <= 96), no host synchronisation. */
size_t gnf4_grouped_gemm_mxfp4_workspace_bytes(int M, int K);
int gnf4_grouped_gemm_mxfp4_native_max_rows(void);
gnf4_status gnf4_grouped_gemm_mxfp4_ws(const void *a, const uint8_t *w, const uint8_t *scales,
                                       const int32_t *offsets, const int32_t *counts, int E, int N, int K, int M,
                                       void *y, void *workspace, size_t workspace_bytes, void *stream);

/* ------------------------------------------------------------------ */
/* Grouped GEMV (decode: at most 8 rows per group)                     */
/* ------------------------------------------------------------------ */

/* Decode variant for a handful of rows per expert (grouped-nf4-gemm
 * index.json, limitations: gemv_mxfp4_b32 "re-streams weights per row: it is
 * a decode lever for a handful of rows").  Here every weight byte is read
 * once for all of its group's rows.  Same arguments and rules as the GEMM
 * calls; additionally every group must hold at most 8 rows (a caller with
 * T <= 8 tokens and distinct experts per token always satisfies this).  A
 * larger group is skipped and flagged with GNF4_DEVERR_GEMV_ROWS. */
gnf4_status gnf4_grouped_gemv_nf4(const void *a, const uint8_t *w, const float *absmax, const int32_t *offsets,
                                  const int32_t *counts, int E, int N, int K, int M, void *y, void *stream);
gnf4_status gnf4_grouped_gemv_mxfp4(const void *a, const uint8_t *w, const uint8_t *scales, const int32_t *offsets,
                                    const int32_t *counts, int E, int N, int K, int M, void *y, void *stream);

/* ------------------------------------------------------------------ */
/* Data gradient of the grouped projection                             */
/* ------------------------------------------------------------------ */

/* dX = dY . W on the same packed stacks the forward call reads
 * (grouped-nf4-gemm index.json, system_manifest.owns: "grouped packed GEMM
 * (NF4 and native MXFP4) and its dgrad"; entrypoints:
 * nf4_grouped:dgrad_4bit_grouped).  For every sorted row r of expert e:
 *     dx[r, k] = sum_n dy[r, n] * dq(W_e)[n, k],
 * fp32 accumulation, bf16 output [M, K].  dy is bf16 [M, N] (the gradient of
 * the forward output), w / scales / offsets / counts exactly as the grouped
 * GEMM calls (same shape rules).  Rows past offsets[E] are not written. */
gnf4_status gnf4_grouped_dgrad_nf4(const void *dy, const uint8_t *w, const float *absmax, const int32_t *offsets,
                                   const int32_t *counts, int E, int N, int K, int M, void *dx, void *stream);
gnf4_status gnf4_grouped_dgrad_mxfp4(const void *dy, const uint8_t *w, const uint8_t *scales, const int32_t *offsets,
                                     const int32_t *counts, int E, int N, int K, int M, void *dx, void *stream);

/* ------------------------------------------------------------------ */
/* Fused gate_up projection + SwiGLU                                   */
/* ------------------------------------------------------------------ */

/* The first projection of the expert MLP with its gated activation in the
 * epilogue (grouped-nf4-gemm releases, v0.2.5 "arena -> kernel":
 * moe_layer_forward runs gate -> GLU -> down; index.json, system_manifest:
 * swiglu is one of the decode glue kernels).  The pages print neither the
 * activation nor the row order; the reading used here: w_gate_up is one
 * stack [E, 2I, K/2] (scales [E, 2I, K/64] fp32 for NF4, [E, 2I, K/32] e8m0
 * for MXFP4) whose rows [0, I) are the gate rows and rows [I, 2I) the up
 * rows, and for every sorted row r of expert e
 *     h[r, i] = silu(g) * u,  g = sum_k a[r,k] W_e[i,k],  u = sum_k a[r,k] W_e[I+i,k],
 *     silu(x) = x / (1 + exp(-x)),
 * with g and u accumulated in fp32 and h rounded once to bf16 [M, I].  The
 * [M, 2I] projection output never reaches global memory.
 *
 * Arguments as the grouped GEMM / GEMV calls, with I (the output width) in
 * place of N: I must be a positive multiple of 64, at most 2^29.  The GEMV forms keep the
 * rule of at most 8 rows per group (larger groups are skipped and flagged
 * with GNF4_DEVERR_GEMV_ROWS). */
gnf4_status gnf4_grouped_gemm_nf4_swiglu(const void *a, const uint8_t *w_gate_up, const float *absmax,
                                         const int32_t *offsets, const int32_t *counts, int E, int I, int K, int M,
                                         void *h, void *stream);
gnf4_status gnf4_grouped_gemm_mxfp4_swiglu(const void *a, const uint8_t *w_gate_up, const uint8_t *scales,
                                           const int32_t *offsets, const int32_t *counts, int E, int I, int K, int M,
                                           void *h, void *stream);
gnf4_status gnf4_grouped_gemv_nf4_swiglu(const void *a, const uint8_t *w_gate_up, const float *absmax,
                                         const int32_t *offsets, const int32_t *counts, int E, int I, int K, int M,
                                         void *h, void *stream);
gnf4_status gnf4_grouped_gemv_mxfp4_swiglu(const void *a, const uint8_t *w_gate_up, const uint8_t *scales,
                                           const int32_t *offsets, const int32_t *counts, int E, int I, int K, int M,
                                           void *h, void *stream);

/* ------------------------------------------------------------------ */
/* Decode GEMV with the top-k combine in its epilogue                  */
/* ------------------------------------------------------------------ */

/* The grouped GEMV of the second projection followed, in the same launch,
 * by the top-k combine (grouped-nf4-gemm index.json, problems_solved[5]:
 * "top-k combine" among the decode tail folded into fewer launches):
 *     y[r, n]   = sum_k a[r, k] * W_e[n, k]            (as gnf4_grouped_gemv_*)
 *     out[t, n] = sum_{j<k} weights[t, j] * y[flat_to_sorted[t*k + j], n]
 * The combine is the same fp32 fmaf sequence as gnf4_combine (slots in
 * order j = 0..k-1, one bf16 rounding), so out equals the unfused
 * GEMV + combine bit for bit.  Pairs whose sorted row is -1 or not below
 * the number of routed rows (offsets[E]) contribute nothing; a token with no
 * such pair gets a zero row.
 *   a, w, scales, offsets, counts, E, N, K, M, y: as gnf4_grouped_gemv_*
 *     (y is still written: the combine reads it);
 *   sorted_to_flat int32 [M] and flat_to_sorted int32 [T*k]: as written by
 *     gnf4_route_permute; weights fp32 [T, k]; out bf16 [T, N];
 *   counters: int32 device memory of gnf4_combine_counters_bytes(T, N)
 *     bytes, zero-filled once by the caller before its first use; every call
 *     that ends without a device error leaves it zero again (so the call is
 *     safe to capture in a CUDA graph).  After a call that set a device
 *     error, zero it again.  Calls that overlap on the GPU need separate
 *     counters. */
size_t gnf4_combine_counters_bytes(int T, int N);
gnf4_status gnf4_grouped_gemv_nf4_combine(const void *a, const uint8_t *w, const float *absmax,
                                          const int32_t *offsets, const int32_t *counts, int E, int N, int K, int M,
                                          void *y, const int32_t *sorted_to_flat, const int32_t *flat_to_sorted,
                                          const float *weights, int T, int k, void *out, int32_t *counters,
                                          void *stream);
gnf4_status gnf4_grouped_gemv_mxfp4_combine(const void *a, const uint8_t *w, const uint8_t *scales,
                                            const int32_t *offsets, const int32_t *counts, int E, int N, int K,
                                            int M, void *y, const int32_t *sorted_to_flat,
                                            const int32_t *flat_to_sorted, const float *weights, int T, int k,
                                            void *out, int32_t *counters, void *stream);

/* The grouped GEMM of the second projection (prefill: any number of rows
 * per group) with the same top-k combine after each work unit's epilogue
 * (grouped-nf4-gemm releases, v0.2.5 "arena -> kernel": moe_layer_forward
 * runs gate -> GLU -> down, then the weighted unsort).  Results, arguments
 * and counter rules exactly as gnf4_grouped_gemv_*_combine (T >= 0, k >= 1,
 * T*k < 2^31 for both), with the shape
 * rules of gnf4_grouped_gemm_*: out equals gnf4_grouped_gemm_* followed by
 * gnf4_combine bit for bit.  y is still written (the combine reads the
 * token's other rows from it through L2).  Each unit's combine runs after
 * its accumulator is released, so it overlaps the next unit's MMAs.  M == 0
 * zeroes out (no pair is valid).  One launch; every group takes the decode
 * path (there is no native-path variant of this call). */
gnf4_status gnf4_grouped_gemm_nf4_combine(const void *a, const uint8_t *w, const float *absmax,
                                          const int32_t *offsets, const int32_t *counts, int E, int N, int K, int M,
                                          void *y, const int32_t *sorted_to_flat, const int32_t *flat_to_sorted,
                                          const float *weights, int T, int k, void *out, int32_t *counters,
                                          void *stream);
gnf4_status gnf4_grouped_gemm_mxfp4_combine(const void *a, const uint8_t *w, const uint8_t *scales,
                                            const int32_t *offsets, const int32_t *counts, int E, int N, int K,
                                            int M, void *y, const int32_t *sorted_to_flat,
                                            const int32_t *flat_to_sorted, const float *weights, int T, int k,
                                            void *out, int32_t *counters, void *stream);

/* ------------------------------------------------------------------ */
/* Native W4A8 mode: MXFP8 activations x MXFP4 weights                 */
/* ------------------------------------------------------------------ */

/* The block-scaled tensor-core form of the MXFP4 projection (bw24 v0.9.0
 * release notes, Documentation "prefill arc design": W4A8-FP8, e4m3
 * activations times native e2m1 weights in one block-scaled MMA; Features
 * "f8f4 tile piece 1": e4m3 activation quantisation; grouped-nf4-gemm
 * index.json, system_manifest.owns: native MXFP4).  The activations are
 * first quantised to MXFP8; the weights are the MXFP4 stack unchanged.
 *
 * gnf4_quantize_mxfp8: x bf16 [M, K] -> codes e4m3 [M, K] (u8) and scales
 * e8m0 [M, K/32] (u8).  Per block of 32 consecutive k of one row:
 *     X = floor(log2(max |x|)) - 8, clamped to [-127, 127] (X = -127 for an
 *         all-zero block); scale byte = X + 127;
 *     code = x * 2^-X rounded to the nearest e4m3 value, ties to even,
 *            saturating at +-448, sign kept on zero results
 * (OCP MX v1.0 MXFP8; the pages give no rule, this is the reading used).
 * Bit-exact: the same inputs give the same bytes on every run.  K must be a
 * positive multiple of 32 and M >= 0 (M == 0 does nothing); inputs must be
 * finite.  x, codes: 16-byte aligned device memory; scales: device memory.
 *
 * gnf4_grouped_gemm_w4a8: for every sorted row r of expert e
 *     y[r, n] = sum_k A[r, k] * W_e[n, k],
 *     A[r, k] = e4m3(codes[r, k]) * 2^(a_scales[r, k/32] - 127),
 *     W_e[n, k] = e2m1(w[e, n, k]) * 2^(w_scales[e, n, k/32] - 127),
 * products exact, fp32 accumulation, bf16 output y [M, N].  w, w_scales,
 * offsets, counts, E, N and M as the MXFP4 grouped GEMM; a_codes / a_scales
 * as written by gnf4_quantize_mxfp8 for the group-sorted rows.  K must be a
 * multiple of 64 in [128, 65536], and E*N < 2^31.  Alignment: a_codes
 * 16 bytes, w 32 bytes, y 16 bytes.  Rows past offsets[E] are not written. */
gnf4_status gnf4_quantize_mxfp8(const void *x, int M, int K, uint8_t *codes, uint8_t *scales, void *stream);

/* Two-term form (the activations as hi + lo, two MXFP8 tensors), which
 * keeps the bf16-activation accuracy of the MXFP4 GEMM on the native path
 * (a reading: no page gives a rule for splitting the activation operand of
 * the block-scaled MXFP4 GEMM).  Per block of 32 consecutive k of one row:
 *     hi = MXFP8 of x, lo = MXFP8 of the exact residual r = x - hi,
 *     both with X = floor(log2(max |value|)) - 7 (one binade of headroom,
 *     so no element saturates), e4m3 round to nearest even;
 * x - (hi + lo) is one e4m3 rounding of r (at most 2^-8 of the block's
 * largest |x|).  Bit-exact.  Buffers as gnf4_quantize_mxfp8, twice.
 *
 * gnf4_grouped_gemm_w4a8x2: y[r, n] = sum_k (hi[r,k] + lo[r,k]) * W_e[n,k],
 * products exact, fp32 accumulation, bf16 output; the hi and lo rows of a
 * group are stacked into one operand, so each block-scaled MMA multiplies
 * both terms.  Arguments and rules as gnf4_grouped_gemm_w4a8, with both
 * terms' codes (16-byte aligned) and scales. */
gnf4_status gnf4_quantize_mxfp8_split(const void *x, int M, int K, uint8_t *hi_codes, uint8_t *hi_scales,
                                      uint8_t *lo_codes, uint8_t *lo_scales, void *stream);
gnf4_status gnf4_grouped_gemm_w4a8x2(const uint8_t *hi_codes, const uint8_t *hi_scales, const uint8_t *lo_codes,
                                     const uint8_t *lo_scales, const uint8_t *w, const uint8_t *w_scales,
                                     const int32_t *offsets, const int32_t *counts, int E, int N, int K, int M,
                                     void *y, void *stream);
gnf4_status gnf4_grouped_gemm_w4a8(const uint8_t *a_codes, const uint8_t *a_scales, const uint8_t *w,
                                   const uint8_t *w_scales, const int32_t *offsets, const int32_t *counts, int E,
                                   int N, int K, int M, void *y, void *stream);

/* Native W4A4 mode: MXFP4 activations x MXFP4 weights on kind::mxf4
 * (the "W4A4" MX mode named next to W4A8; the pages give no rule).
 *
 * gnf4_quantize_mxfp4_act: x bf16 [M, K] -> blocks [M, K/2] (e2m1, element
 * 2i in the low nibble) and scales [M, K/32] (e8m0) by the OCP rule of the
 * weights: X = floor(log2(max |x|)) - 2 clamped to [-127, 127] (-127 for an
 * all-zero block), code = x * 2^-X rounded to the nearest e2m1 value, ties
 * to even, saturating at +-6.  Bit-exact.  K % 32 == 0; x 16-byte and
 * blocks 4-byte aligned.
 *
 * gnf4_grouped_gemm_w4a4: y[r, n] = sum_k A[r, k] * W_e[n, k] with A and W
 * both e2m1 x 2^(scale - 127); products exact, fp32 accumulation, bf16
 * output.  K must be a multiple of 64 in [256, 65536]; a_blocks and w
 * 16-byte aligned, y 16-byte aligned; other rules as gnf4_grouped_gemm_w4a8.
 * The result carries the e2m1 rounding of the activations: against bf16
 * activations each activation moves by at most |a|/3 + 2^(X-2). */
gnf4_status gnf4_quantize_mxfp4_act(const void *x, int M, int K, uint8_t *blocks, uint8_t *scales, void *stream);
gnf4_status gnf4_grouped_gemm_w4a4(const uint8_t *a_blocks, const uint8_t *a_scales, const uint8_t *w,
                                   const uint8_t *w_scales, const int32_t *offsets, const int32_t *counts, int E,
                                   int N, int K, int M, void *y, void *stream);

/* ------------------------------------------------------------------ */
/* Top-k combine                                                       */
/* ------------------------------------------------------------------ */

/* Weighted scatter of expert outputs back to tokens (grouped-nf4-gemm
 * index.json, problems_solved[5] "top-k combine"; releases v0.2.6: the
 * caller's "weighting, unsorting"):
 *   out[t, n] = sum_{j<k} weights[t, j] * y[flat_to_sorted[t*k + j], n],
 * summed in fp32 in order j = 0..k-1, rounded to bf16; pairs whose
 * flat_to_sorted is -1 (or not below T*k) contribute nothing.
 *   y bf16 [T*k, N] (group-sorted expert outputs); flat_to_sorted int32 [T*k];
 *   weights fp32 [T, k]; out bf16 [T, N] OUT.
 * Rules: T >= 0, k >= 1, T*k < 2^31, N >= 8 and N % 8 == 0, y and out
 * 16-byte aligned. */
gnf4_status gnf4_combine(const void *y, const int32_t *flat_to_sorted, const float *weights, int T, int k, int N,
                         void *out, void *stream);

/* ------------------------------------------------------------------ */
/* Decode checks (test support)                                        */
/* ------------------------------------------------------------------ */

/* fp32 decode of `rows` packed rows of K elements: out[r, k] = NF4[code] *
 * absmax[r, k/64] (one fp32 multiply, round to nearest, no flush to zero).
 * This is the reference decode the pages call dequant_ref (grouped-nf4-gemm
 * 0.33.1 on PyPI, example 1).  Rules: K >= 64 and K % 64 == 0, rows >= 0. */
gnf4_status gnf4_dequant_nf4_f32(const uint8_t *w, const float *absmax, int64_t rows, int K, float *out,
                                 void *stream);

/* fp32 decode of MXFP4 rows: out[r, k] = e2m1[code] * 2^(scale-127), with
 * scale 255 decoding to NaN (same page, example 2).  Rules: K >= 32 and
 * K % 32 == 0, rows >= 0. */
gnf4_status gnf4_dequant_mxfp4_f32(const uint8_t *w, const uint8_t *scales, int64_t rows, int K, float *out,
                                   void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GNF4_H */

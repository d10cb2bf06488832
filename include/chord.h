/*
 * chord.h -- C ABI of the B200 (sm_100a) W4A16 mixture-of-experts layer.
 *
 * The layer (Novita/vLLM blog "vLLM x Novita AI: Chord W4A16 INT4 MoE Kernel fuer
 * Kimi K2.x"; sections cited below by their headings) takes BF16 activations, uint4
 * weights packed eight per int32 along K, and one BF16 scale per 32 consecutive K
 * elements of each output row ("vLLM-Integration": uint4, group-32, BF16 scales). A
 * weight element is w = bf16((q - 8) * s), subtract first, then scale, rounded once to
 * BF16 ("H200 und Blackwell indexierter Decode").
 *
 *   out[t] = sum over local top-k slots j of  topk_weights[t,j] * W2[e] . act(W13[e] . x[t])
 *   act(h) = silu(h[0:I]) * h[I:2I]      (rounded to BF16 before the down projection)
 *
 * with FP32 accumulation throughout (F16 accumulation is not offered; "vLLM-Integration",
 * deployment notes).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer argument named as "device" is a CUDA device pointer owned by the
 *    caller. The library allocates no device or host memory on any call.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL means the legacy default
 *    stream) and returns before it runs. No entry point reads device memory back to
 *    the host, so align + forward can be captured in a CUDA graph ("vLLM-Integration":
 *    the indexed fast path consumes over-allocated routing buffers without reading the
 *    routed count back to the host).
 *  - Argument errors are detected on the host before anything is enqueued and returned
 *    as a chord_status_t; chord_last_error_detail() then describes the failure (the
 *    text is thread-local and valid until the next call on the same thread).
 *  - Errors found on the device (routing validation, weight-blob header mismatch, a
 *    bounded wait that gave up) are OR-ed into a status word inside the forward
 *    workspace and read with chord_moe_check_status().
 *  - Device code is built for sm_100a only. On any other device the entry points that
 *    launch work return CHORD_ERR_UNSUPPORTED.
 */
#ifndef CHORD_H_
#define CHORD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define CHORD_API __attribute__((visibility("default")))
#else
#define CHORD_API
#endif

typedef struct CUstream_st* chord_stream_t; /* identical to cudaStream_t */

typedef enum {
  CHORD_OK = 0,
  CHORD_ERR_INVALID_ARG = 1,        /* null pointer, negative or inconsistent size */
  CHORD_ERR_UNSUPPORTED = 2,        /* group size != 32, unsupported shape, not sm_100 */
  CHORD_ERR_LAYOUT_MISMATCH = 3,    /* weight blob of another role/shape/layout */
  CHORD_ERR_WORKSPACE_TOO_SMALL = 4,
  CHORD_ERR_CUDA = 5,               /* a CUDA runtime call failed (see detail text) */
  CHORD_ERR_DEVICE = 6              /* chord_moe_check_status found device status bits */
} chord_status_t;

/* Device status bits (chord_moe_check_status). */
#define CHORD_DEV_ROUTING_INVALID 0x1u /* VALIDATE_ROUTING found inconsistent routing */
#define CHORD_DEV_BLOB_MISMATCH   0x2u /* a weight blob header does not match the call */
#define CHORD_DEV_TIMEOUT         0x4u /* a bounded on-chip wait gave up */
#define CHORD_DEV_BLOCK_M_MISMATCH 0x8u /* routing tensors built for another block_m: nothing computed */

/* The routing tag: word [1] of num_tokens_padded, written by every routing entry point
 * (chord_moe_align, chord_moe_align_noalloc, chord_router_topk_align) and checked on the
 * device by chord_moe_forward before it reads expert_ids. A producer of routing tensors
 * other than this library must write it too. */
#define CHORD_ROUTING_TAG(block_m) ((int32_t)(0x52540000u | (uint32_t)(block_m)))

/* Bytes at the start of a forward or grouped workspace that the caller zeroes once after
 * allocating it (status word and stream-K flags); the library keeps them consistent. */
#define CHORD_WORKSPACE_HEADER_BYTES 65536

/* Weight roles for chord_repack_weights. */
#define CHORD_ROLE_GATE_UP 1 /* W13 [E, 2I, H]: rows [0,I) gate, rows [I,2I) up */
#define CHORD_ROLE_DOWN    2 /* W2  [E, H, I] */
#define CHORD_ROLE_GROUPED_CONTIGUOUS 3 /* W [E, N, K] for chord_grouped_contiguous */
#define CHORD_ROLE_GROUPED_MASKED     4 /* W [E, N, K] for chord_grouped_masked */

/* Flags for chord_moe_forward. */
#define CHORD_FLAG_VALIDATE_ROUTING 0x1 /* check routing tensors on the device first */
#define CHORD_FLAG_FORCE_STREAM     0x2 /* force the weight-streaming (decode) schedule */
#define CHORD_FLAG_FORCE_TENSOR     0x4 /* force the tensor-core (prefill) schedule */
#define CHORD_FLAG_OUTPUT_FP32      0x8 /* `out` is float [T, H]: the FP32 sums before the final
                                           BF16 rounding (a tensor-parallel rank's partial) */

CHORD_API const char* chord_status_string(int status);
CHORD_API const char* chord_last_error_detail(void);

/* ------------------------------------------------------------------------------------
 * Routing sort ("Zwei Kernel-Familien": the indexed family consumes vLLM's
 * sorted_ids / expert_ids / num_tokens_padded; Figure 3: activations stay unpadded and
 * the routing indices carry padding sentinels).
 *
 * Flat slot index f = t*topk + j. A slot is local when 0 <= topk_ids[f] < E; any other
 * id (-1, or a global id of an expert on another shard) is skipped. With c_e the local
 * slots of expert e, p_e = ceil(c_e / block_m) * block_m and off_e = sum_{e' < e} p_e':
 *   sorted_ids[off_e + r] = the r-th local flat index of expert e, in increasing f;
 *   every other entry of sorted_ids (up to the capacity below) = T*topk (sentinel);
 *   expert_ids[b] = e for the p_e / block_m blocks of expert e, in increasing e, and
 *   -1 for every block at or past num_tokens_padded / block_m;
 *   num_tokens_padded[0] = off_E;   expert_offsets[e] = off_e for e in [0, E].
 *   num_tokens_padded[1] = CHORD_ROUTING_TAG(block_m): the block_m these tensors were
 *   built for, which chord_moe_forward checks on the device (the padded count alone does
 *   not reveal it, and a forward with another block_m would misread expert_ids).
 * An expert with no local slot gets no block. The result is deterministic.
 *
 * Capacities: sorted_ids holds chord_moe_align_capacity() int32, expert_ids holds
 * chord_moe_align_num_blocks() int32. Limits: 1 <= E <= 1024, 1 <= block_m <= 256,
 * capacity < 2^31. `workspace` (device, >= chord_moe_align_workspace_bytes() bytes,
 * any content, 256-byte aligned) is scratch for large T*topk; it may be NULL when
 * that size is 0. expert_offsets (device, E+1 int32) may be NULL.
 * ---------------------------------------------------------------------------------- */
CHORD_API int64_t chord_moe_align_capacity(int64_t T, int topk, int E, int block_m);
CHORD_API int64_t chord_moe_align_num_blocks(int64_t T, int topk, int E, int block_m);
CHORD_API size_t chord_moe_align_workspace_bytes(int64_t T, int topk, int E);
CHORD_API chord_status_t chord_moe_align(const int32_t* topk_ids /* device [T, topk] */, int64_t T,
                               int topk, int E, int block_m, int32_t* sorted_ids,
                               int32_t* expert_ids, int32_t* num_tokens_padded /* [2] */,
                               int32_t* expert_offsets /* [E+1] or NULL */, void* workspace,
                               size_t workspace_bytes, chord_stream_t stream);

/* ----------------------------------------------------------------------------------
 * chord_router_topk_align: the router step upstream of moe_align, fused with it.
 *
 * The layer's problem statement routes by top-k softmax with the weights renormalised
 * over the chosen experts; the Chord blog leaves routing outside its kernel timings
 * ("Messungen") and feeds the indexed path vLLM's sorted routing ("Zwei
 * Kernel-Familien"). Per token t:
 *   topk_ids[t, r]     = the expert with the r-th largest logit (r = 0 .. topk-1), ties to
 *                        the lower expert id; GLOBAL ids in [0, E_global);
 *   topk_weights[t, r] = exp(l_r - l_0) / sum_j exp(l_j - l_0), i.e. the softmax over all
 *                        logits renormalised over the chosen ones (fp32);
 * then exactly the routing tensors of chord_moe_align(topk_ids, T, topk, E, block_m, ...)
 * for the local experts [0, E) (ids >= E belong to other shards).
 *
 * logits: device fp32 [T, E_global], finite or -inf. topk_ids / topk_weights: device
 * [T, topk] int32 / fp32 outputs. The other arguments, limits and the workspace rule are
 * those of chord_moe_align, plus topk <= E_global <= 1024. Up to 8 tokens run as ONE
 * launch (the CTA that routes the tokens also sorts them); larger batches run a routing
 * kernel (one warp per token) and the sort kernels. Returns CHORD_ERR_UNSUPPORTED for
 * E_global out of range.
 * ---------------------------------------------------------------------------------- */
CHORD_API chord_status_t chord_router_topk_align(const float* logits, int64_t T, int E_global, int topk, int E,
                                                 int block_m, int32_t* topk_ids, float* topk_weights,
                                                 int32_t* sorted_ids, int32_t* expert_ids,
                                                 int32_t* num_tokens_padded /* [2] */,
                                                 int32_t* expert_offsets /* [E+1] or NULL */, void* workspace,
                                                 size_t workspace_bytes, chord_stream_t stream);

/* Routing sort for callers that cannot allocate device memory (no counterpart on the
 * pages). Same arguments, results and limits as chord_moe_align, minus the workspace:
 * the scratch that large batches need lives in a static device array of 576 KiB that
 * every GPU loading this library holds until the process exits. Made for callers that
 * may not call cudaMalloc where they route a batch, e.g. a serving engine that reserved
 * all free device memory up front, or code running under stream capture without a
 * workspace tensor at hand.
 *  - T*topk must be <= 131072 (2^17); larger batches return CHORD_ERR_UNSUPPORTED.
 *  - Allocates nothing. The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, once per device); make that first call before any stream
 *    capture.
 *  - All calls share the array. Nothing in it needs to start at zero (each call
 *    overwrites every entry it later reads), but calls that overlap on the GPU (other
 *    streams, other host threads) race on it: serialise them.
 * Returns the status chord_moe_align returns for the same arguments (with the same
 * chord_last_error_detail() text), plus CHORD_ERR_UNSUPPORTED with a detail naming the
 * limit when T*topk exceeds 2^17, and CHORD_ERR_CUDA when the address lookup fails. */
CHORD_API chord_status_t chord_moe_align_noalloc(const int32_t* topk_ids, int64_t T, int topk, int E,
                                                 int block_m, int32_t* sorted_ids, int32_t* expert_ids,
                                                 int32_t* num_tokens_padded, int32_t* expert_offsets,
                                                 chord_stream_t stream);

/* ------------------------------------------------------------------------------------
 * One-time weight repack ("Gruppierte SM90-Kernel": prepared weights are permuted INT4
 * buffers with re-laid scales, and the mode is recorded in the prepared weight and
 * checked at dispatch; Figure 2: layouts are fixed at model load).
 *
 * In:  qweight (device) int32 [E, N, K/8]: code of (n, k) in bits 4*(k%8)..+3 of word
 *      [n, k/8] (low nibble first); scales (device) bf16 bits [E, N, K/32].
 *      For CHORD_ROLE_GATE_UP, N = 2*I with gate rows first; for CHORD_ROLE_DOWN, N = H.
 * Out: `out` (device, >= chord_repacked_bytes() bytes, 256-byte aligned): an opaque
 *      blob = 256-byte header (magic, version, role, E, N, K, group) + codes + scales
 *      in the tile layout the forward kernels read (128 rows x 128 K per tile; gate and
 *      up rows interleaved in blocks of 8 for CHORD_ROLE_GATE_UP).
 * Requires group_size == 32 (else CHORD_ERR_UNSUPPORTED), N % 128 == 0, K % 128 == 0.
 * The input buffers may be freed once the stream has run the repack.
 * ---------------------------------------------------------------------------------- */
CHORD_API size_t chord_repacked_bytes(int E, int N, int K, int group_size);
CHORD_API chord_status_t chord_repack_weights(const int32_t* qweight, const uint16_t* scales, int E,
                                    int N, int K, int group_size, int role, void* out,
                                    size_t out_bytes, chord_stream_t stream);

/* Inverse layout, for checks: blob -> logical-order bf16 weights w[E, N, K] computed
 * with the forward kernels' own dequantisation (rows in the caller's logical order).
 * w_bf16: device, E*N*K uint16. */
CHORD_API chord_status_t chord_dequant_weights(const void* blob, size_t blob_bytes, uint16_t* w_bf16,
                                     chord_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Schedule selector ("Kernel-Optimierungen": the tokens routed per expert, tok_e, not
 * the total token count, decide the schedule; below ~80 tokens per expert the indexed
 * resolver keeps a block-count search, above it sizes block_m around each expert's
 * padded rows). Host-only and memoised. Returns the block_m to pass to
 * chord_moe_align and chord_moe_forward. Small values (<= 32) select the
 * weight-streaming schedule in chord_moe_forward, larger ones the tensor-core
 * schedule. tok_e is estimated without reading routing back: T*topk / E_global.
 * ---------------------------------------------------------------------------------- */
CHORD_API int chord_select_block_m(int64_t T, int topk, int E_local, int E_global, int H, int I);

/* ------------------------------------------------------------------------------------
 * The layer.
 *
 * hidden       device bf16 [T, H]
 * topk_ids     device int32 [T, topk] (same convention as chord_moe_align)
 * topk_weights device fp32  [T, topk]; not renormalised over local slots
 * sorted_ids, expert_ids, num_tokens_padded: device routing tensors for this block_m
 *              (from chord_moe_align or any producer with the same contract; entries
 *              >= T*topk are padding, blocks with expert_ids outside [0,E) are skipped).
 *              num_tokens_padded[1] must be CHORD_ROUTING_TAG(block_m); otherwise the
 *              kernels read no other routing tensor, compute nothing, write zero rows
 *              to `out` and set CHORD_DEV_BLOCK_M_MISMATCH (checked on the device, so a
 *              captured graph needs no readback).
 * w13, w2      device blobs from chord_repack_weights (roles GATE_UP [E,2I,H], DOWN [E,H,I])
 * out          device bf16 [T, H]; every row is written (0 for tokens with no local slot)
 * workspace    device, >= chord_moe_workspace_bytes(), 256-byte aligned. Its first
 *              CHORD_WORKSPACE_HEADER_BYTES hold the device status word (offset 0) and the
 *              flags with which the weight-streaming GEMM's stream-K workers hand partial
 *              sums to one another (each flag is reset by its reader): zero them once after
 *              allocating, and again after a call that raised CHORD_DEV_TIMEOUT (its
 *              flags may be left set). The rest is scratch that needs no initialisation.
 *
 * Requires H % 128 == 0, I % 128 == 0, 1 <= block_m <= 256 (same as used for align).
 * Concurrent forwards must not share a workspace.
 * ---------------------------------------------------------------------------------- */
CHORD_API size_t chord_moe_workspace_bytes(int64_t T, int topk, int E, int H, int I, int block_m);
CHORD_API chord_status_t chord_moe_forward(const uint16_t* hidden, const int32_t* topk_ids,
                                 const float* topk_weights, const int32_t* sorted_ids,
                                 const int32_t* expert_ids, const int32_t* num_tokens_padded,
                                 int block_m, const void* w13, const void* w2, int64_t T,
                                 int H, int I, int E, int topk, uint16_t* out, void* workspace,
                                 size_t workspace_bytes, int flags, chord_stream_t stream);

/* Synchronises `stream`, copies the workspace status word to *device_status, clears it
 * on the device, and returns CHORD_OK when it was zero, else CHORD_ERR_DEVICE. */
CHORD_API chord_status_t chord_moe_check_status(void* workspace, chord_stream_t stream,
                                      uint32_t* device_status);

/* ------------------------------------------------------------------------------------
 * Grouped operators ("Gruppierte SM90-Kernel": the second operator family, with its own
 * routing layouts; "Gruppierte Operatoreintrittspunkte": contiguous for prefill, masked
 * for decode). Each computes, for every row m of x that belongs to an expert e_m,
 *     out[m, n] = bf16_rne( sum_k x[m, k] * w[e_m][n, k] ),  w = bf16((q - 8) * s),
 * with FP32 accumulation (the dequantisation of the indexed path). Rows that belong to
 * no expert are not written: the caller ignores them.
 *
 * chord_grouped_contiguous: rows concatenated by expert, each expert's run padded to a
 *   multiple of 128 rows ("Kontiguoeser Prefill").
 *   x         device bf16 [M, K], 16-byte aligned
 *   m_indices device int32 [M], 16-byte aligned: the expert of each row in [0, E), or
 *             a negative id for padding.
 *             Every aligned 128-row block (rows 128b .. 128b+127) must hold rows of at
 *             most one expert; a block that mixes experts or names an id >= E is not
 *             computed and sets CHORD_DEV_ROUTING_INVALID in the workspace status.
 *   out       device bf16 [M, N], 16-byte aligned
 * chord_grouped_masked: a fixed row budget per expert ("Maskierter Decode").
 *   x         device bf16 [E, max_m, K] (= [E * max_m, K]), 16-byte aligned
 *   masked_m  device int32 [E]: the valid rows of each expert; rows m with
 *             m % max_m >= masked_m[m / max_m] are not written. Counts outside
 *             [0, max_m] are clamped and set CHORD_DEV_ROUTING_INVALID.
 *   expected_m host hint (> 0), the rows per expert the caller expects; it only picks
 *             the schedule and never changes results.
 *   out       device bf16 [E * max_m, N] (flat even when x is 3-D)
 * Both: w is a blob from chord_repack_weights with the matching role
 *   (CHORD_ROLE_GROUPED_CONTIGUOUS / CHORD_ROLE_GROUPED_MASKED) and shape [E, N, K]; a
 *   blob of another role or shape fails with CHORD_ERR_LAYOUT_MISMATCH (prepared in this
 *   process) or sets CHORD_DEV_BLOB_MISMATCH (foreign blob: the kernel reads its
 *   header). N % 128 == 0, K % 128 == 0, 1 <= E <= 1024.
 *   workspace: device, >= chord_grouped_workspace_bytes(rows, E) bytes, rows = M or
 *   E * max_m, 256-byte aligned; its first CHORD_WORKSPACE_HEADER_BYTES hold the status
 *   word and the stream-K flags as for chord_moe_forward (zero once; read the status with
 *   chord_moe_check_status).
 *   flags: CHORD_FLAG_FORCE_STREAM / CHORD_FLAG_FORCE_TENSOR pick the schedule; by
 *   default expected rows per expert (M / E, or expected_m) <= 16 streams the weights.
 *   Two kernels run on `stream`: a routing pass over m_indices / masked_m, then the GEMM;
 *   nothing is read back to the host, so both calls can be captured in a CUDA graph.
 * ---------------------------------------------------------------------------------- */
CHORD_API size_t chord_grouped_workspace_bytes(int64_t rows, int E);
CHORD_API chord_status_t chord_grouped_contiguous(const uint16_t* x, int64_t M, int K, const int32_t* m_indices,
                                                  const void* w, int E, int N, uint16_t* out, void* workspace,
                                                  size_t workspace_bytes, int flags, chord_stream_t stream);
CHORD_API chord_status_t chord_grouped_masked(const uint16_t* x, int E, int64_t max_m, int K,
                                              const int32_t* masked_m, int64_t expected_m, const void* w, int N,
                                              uint16_t* out, void* workspace, size_t workspace_bytes, int flags,
                                              chord_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Exchange steps of sharded deployments. The Chord blog runs the layer as expert-parallel
 * (EP8/EP16/EP32) and tensor-parallel (TP8 single-instance) shards ("TL;DR";
 * "vLLM-Integration": the h200_tp8 profile) and leaves the communication out of its
 * kernel timings ("Messungen"). These entry points are the device steps around the
 * collectives; the collectives themselves (all-to-all, all-reduce) are the caller's.
 *
 * Expert parallel, W ranks, rank d owning global experts [d*E_rank, (d+1)*E_rank):
 *  chord_ep_plan: for this rank's T tokens and their GLOBAL topk_ids [T, topk] (ids outside
 *    [0, W*E_rank) are dropped), one send row per (token t, rank d) such that t has at
 *    least one slot on d. send_rows[i] = t*W + d for the i-th send row, rows grouped by
 *    d in increasing d and by t in increasing t inside each group; rank_offsets[d] = the
 *    first row of rank d, rank_offsets[W] = the row count (the caller reads the W + 1
 *    offsets back to size its all-to-all); row_of[t*W + d] = -1 for every pair (set here,
 *    filled by chord_ep_pack). send_rows: device int32 [T*W]; rank_offsets: device int32
 *    [W+1]; row_of: device int32 [T*W]; workspace: device, >= chord_ep_plan_workspace_bytes,
 *    256-byte aligned, scratch. Limits: 1 <= W <= 64, W*E_rank <= 4096, T*W < 2^31.
 *  chord_ep_pack: the send buffers of those rows: send_x[i] = hidden[t] (bf16 [rows, H]),
 *    send_ids[i, j] = topk_ids[t, j] - d*E_rank when slot j is on rank d, else -1, and
 *    send_w[i, j] = topk_weights[t, j] for those slots, else 0; row_of[t*W + d] = i. The
 *    receiving rank runs chord_moe_align + chord_moe_forward on the rows it receives (with
 *    send_ids as topk_ids over its E_rank experts) and returns one bf16 output row per row.
 *    send_x: device bf16 [T*W, H] (capacity), send_ids int32 / send_w fp32 [T*W, topk];
 *    hidden and send_x 16-byte aligned, H % 8 == 0.
 *  chord_ep_combine: out[t] = bf16( sum over d = 0 .. W-1 with a row i = row_of[t*W + d]
 *    of float(back[i]) ), the sum in FP32 in increasing d; 0 for a token with no slot on
 *    any rank. back: device bf16 [rows, H], the returned rows in send-row order; out:
 *    device bf16 [T, H]; both 16-byte aligned.
 * Tensor parallel, each rank holding a slice of every expert's intermediate dimension:
 *  chord_moe_forward with CHORD_FLAG_OUTPUT_FP32 writes the rank's FP32 partial output,
 *  the caller all-reduces the partials (sum), and chord_round_bf16 rounds the total once:
 *  out[i] = bf16_rne(in[i]) for i < n (device float in, device bf16 out).
 *  chord_tp_reduce_round does the all-reduce and the rounding in one pass over the ranks'
 *  buffers by pointer (peer memory mapped into this process, e.g. over NVLink; or W
 *  buffers of one GPU standing in for the ranks): rank `rank` of W takes the slice of
 *  4-float vectors [rank*n/4/W, (rank+1)*n/4/W) and writes outs[d][i] = bf16_rne(
 *  partials[0][i] + partials[1][i] + ... + partials[W-1][i]) (FP32 sums in rank order, so
 *  every output holds the same bits) into every rank d's output. partials: W device
 *  pointers to float [n] (16-byte aligned), outs: W device pointers to bf16 [n] (8-byte
 *  aligned); both pointer arrays are host memory, read during the call. n % 4 == 0,
 *  1 <= W <= 64. The caller orders the ranks: every partial is complete before any
 *  rank's call runs, and an output is complete once every rank's call has run (a barrier
 *  on each side).
 * All are asynchronous on `stream`; argument errors return before anything is enqueued.
 * ---------------------------------------------------------------------------------- */
CHORD_API size_t chord_ep_plan_workspace_bytes(int64_t T, int W);
CHORD_API chord_status_t chord_ep_plan(const int32_t* topk_ids, int64_t T, int topk, int E_rank, int W,
                                       int32_t* send_rows, int32_t* rank_offsets, int32_t* row_of, void* workspace,
                                       size_t workspace_bytes, chord_stream_t stream);
CHORD_API chord_status_t chord_ep_pack(const uint16_t* hidden, const int32_t* topk_ids, const float* topk_weights,
                                       int64_t T, int H, int topk, int E_rank, int W, const int32_t* send_rows,
                                       const int32_t* rank_offsets, int32_t* row_of, uint16_t* send_x,
                                       int32_t* send_ids, float* send_w, chord_stream_t stream);
CHORD_API chord_status_t chord_ep_combine(const uint16_t* back, const int32_t* row_of, int64_t T, int H, int W,
                                          uint16_t* out, chord_stream_t stream);
CHORD_API chord_status_t chord_round_bf16(const float* in, int64_t n, uint16_t* out, chord_stream_t stream);
CHORD_API chord_status_t chord_tp_reduce_round(const float* const* partials, uint16_t* const* outs, int W, int rank,
                                               int64_t n, chord_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Measurement hooks (no counterpart on the pages; used by the benchmark).
 *
 * chord_set_timing_events: while set (n == 4), every chord_moe_forward made on the
 * calling thread records the caller-owned cudaEvent_t handles events[0..3] on its
 * stream: [0] right before the gate_up GEMM kernel (after routing validation and, on
 * the tensor-core schedule, the row permutation), [1] between the gate_up and down GEMM
 * kernels, [2] after the down GEMM, [3] after the combine. The grouped operators record
 * [0] right before their GEMM kernel and [1] after it. Records use cudaEventRecordExternal,
 * so a forward captured into a CUDA graph records them when the graph is replayed. n == 0 clears the hook. The handles must stay
 * valid while set. Returns CHORD_ERR_INVALID_ARG for other n or null handles.
 * Without the hook, the layer's GEMM and combine kernels on the weight-streaming schedule
 * are launched early (programmatic dependent launch: each waits on the device for the
 * previous kernel's output); an event between two kernels orders them fully, so while the
 * hook is set they are launched plainly.
 *
 * chord_launch_count: number of CUDA kernels this library has launched in the process
 * (all entry points, all threads), for checking launch counts of a timed region.
 * ---------------------------------------------------------------------------------- */
CHORD_API chord_status_t chord_set_timing_events(void* const* events, int n);
CHORD_API uint64_t chord_launch_count(void);

/* ------------------------------------------------------------------------------------
 * chord_selftest_wait_timeout (diagnostics, no counterpart on the pages): checks the
 * bounded on-chip wait that every pipeline wait of the GEMM kernels uses, without a
 * fault. One CTA waits on an mbarrier that nothing ever completes:
 *   - one thread with a limit of limit_us microseconds (1 .. 1000000): it gives up,
 *     ORs CHORD_DEV_TIMEOUT into *status and raises the CTA's abort flag;
 *   - a second thread with the kernels' own limit (1 s): it sees the abort flag and
 *     returns early, as the other waiters of a GEMM CTA do.
 * status: device uint32, OR-ed (bit 31 would mean the never-completed phase completed);
 * elapsed_ns: device uint64[2], the time each of the two threads waited. Asynchronous on
 * `stream`. Returns CHORD_ERR_INVALID_ARG for null pointers or a limit out of range.
 * ---------------------------------------------------------------------------------- */
CHORD_API chord_status_t chord_selftest_wait_timeout(uint32_t* status, uint64_t* elapsed_ns, uint32_t limit_us,
                                                     chord_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* CHORD_H_ */

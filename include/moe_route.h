/*
 * moe_route.h -- C ABI of libmoe_route.so, the B200 (sm_100a) MoE token-routing library.
 *
 * The routing path of a Mixture-of-Experts layer, one call per stage:
 *   moe_topk_softmax   fused softmax + top-k gating over router logits
 *   moe_align_permute  per-expert histogram, block-padded prefix and stable
 *                      placement of the routed slots (with expert-parallel remap)
 *   moe_gather         activation permute-gather into the expert-grouped layout
 *   moe_combine        top-k weighted combine back to token order
 * Between moe_gather and moe_combine the caller runs its expert MLPs on the
 * expert-grouped rows; they are not part of this library.  Under expert
 * parallelism, moe_reduce_partials sums the ranks' partial combines.
 *
 * Sources (web pages, by title and section):
 *   "project_6/upstream_ref -- Upstream Reference: Deep-Spark xllm + vllm":
 *     "Call Chain: MoE topk_softmax on BI-V100" (topk_softmax as a standalone op,
 *     and a CUDA .so loaded through ctypes as a boundary) and "File Index"
 *     (moe_topk_softmax_kernels.cuh "fused softmax+topk"; moe_align_sum_kernels.cu
 *     "block alignment for scatter"; fused_moe.cpp "gate -> topk -> expand ->
 *     gemm1 -> act -> gemm2 -> combine").
 *   "b70-optimization-lab: 2026-07-16 MTP1 M=2 compact scheduler closure note":
 *     scheduler paragraph (per local expert row count and remapped-row prefix
 *     derived from topk_ids plus expert_map; 8-row tiles owned by occurrences
 *     0 and 8 in the all-duplicate case) and coverage paragraph (a valid
 *     all-remote expert-parallel rank; bitwise-exact checks).
 *
 * Kernel launches use programmatic dependent launch: each kernel lets the next kernel in the
 * stream be scheduled early and waits (griddepcontrol.wait) for the previous one before reading
 * its outputs.  A caller kernel launched right after one of these with programmatic stream
 * serialisation must likewise wait before reading their outputs; ordinary launches need nothing.
 *
 * Conventions shared by every entry point
 *   Notation: T tokens, E (= E_global) experts, E_local experts on this rank,
 *   k experts per token, H hidden size, bs block size.  Slot s = t*k + j is the
 *   j-th routed choice of token t (P = T*k slots).
 *   Memory: every pointer argument is DEVICE memory owned by the caller, except
 *   the host out-parameter of moe_read_status and the host pointer array of
 *   moe_reduce_partials.  All arrays are dense row-major.
 *   The library allocates nothing and never synchronises the stream except in
 *   moe_read_status.  It keeps no global state, with one exception:
 *   moe_align_permute_noalloc keeps its scratch in a fixed 1 MiB device array per
 *   GPU and the array's device address per CUDA context (see that entry point).
 *   Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream).  Every call only enqueues work on it and returns.
 *   Errors: arguments are validated on the host before anything is enqueued;
 *   a non-MOE_OK return means nothing was enqueued (except MOE_ERR_CUDA, which
 *   reports a launch failure).  Conditions only the device can see (an expert
 *   id out of range, a row index past the capacity) are recorded in a caller-
 *   provided device status word (first error wins) and the offending element is
 *   skipped, never dereferenced; read it with moe_read_status.
 *   Alignment: bf16/fp32 tensors are read and written with 16-byte vector
 *   accesses, so moe_gather and moe_combine require 16-byte aligned pointers and
 *   H % 8 == 0.
 *   Sizes: T*k < 2^30 and the align capacity < 2^31 (int32 row and slot ids).
 */
#ifndef MOE_ROUTE_H_
#define MOE_ROUTE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, negative size, k > E, misalignment, ... */
  MOE_ERR_UNSUPPORTED = 2,   /* valid but beyond the library's limits: E > 1024, k > 32, E_local > 1024 */
  MOE_ERR_WORKSPACE = 3,     /* workspace null or smaller than moe_align_workspace_bytes() */
  MOE_ERR_CUDA = 4,          /* a CUDA launch or copy failed */
  MOE_ERR_TIMEOUT = 5,       /* device: a bounded wait ran out (recorded in the status word) */
  MOE_ERR_BAD_EXPERT_ID = 6, /* device: an id outside [0,E) or a map value outside [-1,E_local);
                                the slot was treated as remote */
  MOE_ERR_BAD_ROW = 7        /* device: an inv_perm row outside [-1, capacity); the slot was skipped */
} moe_status_t;

typedef enum { MOE_DTYPE_F32 = 0, MOE_DTYPE_BF16 = 1 } moe_dtype_t;

/* flags */
#define MOE_RENORMALIZE 1u     /* moe_topk_softmax: renormalise the k weights to sum to 1 */
#define MOE_GATHER_ZERO_PAD 2u /* moe_gather: write +0 into the pad rows below N_pad */
#define MOE_GATHER_HIDDEN_READY 4u /* moe_gather: `hidden` was complete before the previous kernel in
                                      the stream was launched, so it may be read before waiting for
                                      that kernel (true when hidden is an input of the routing step) */
#define MOE_SCORING_SIGMOID 16u /* moe_topk_softmax, moe_route_dispatch: score each selected expert
                                   with the logistic function 1/(1+exp(-x)) instead of the softmax
                                   (the sigmoid variant of the gating); the selection is the same */
#define MOE_DISPATCH_GIVEN_IDS 8u /* moe_route_dispatch: topk_ids is an input (routes chosen by the
                                     caller); no gating, logits and topk_weights are not accessed */

/* Human-readable name of a status code (static string, never NULL). */
MOE_API const char* moe_status_string(moe_status_t status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
MOE_API int32_t moe_version(void);

/*
 * moe_topk_softmax -- fused softmax + top-k gating ("Upstream Reference", "File
 * Index": moe_topk_softmax_kernels.cuh, vLLM topk_softmax_kernels.cu).
 *   logits        [T, E] bf16 or fp32 (dtype), row-major, row stride E.
 *   topk_ids      [T, k] int32 out: the k experts with the largest logits, in
 *                 descending logit order; equal logits go to the lower index.
 *   topk_weights  [T, k] fp32 out: softmax over all E logits of the selected
 *                 experts; with MOE_RENORMALIZE divided by their sum instead
 *                 (equivalently exp(x_j - max) / sum over the k selected).
 *                 With MOE_SCORING_SIGMOID ("File Index": moe_topk_sigmoid_kernels.cuh,
 *                 the sigmoid variant, chosen by the moe_fused_topk.cu dispatcher):
 *                 1 / (1 + exp(-x_j)) per selected expert, with MOE_RENORMALIZE
 *                 divided by their sum (1/k if that sum is 0).
 *   Computed in fp32 on the device (exp, sums, one division); within 2e-6 of the
 *   double-precision result.  Selection compares the logits exactly.
 *   Preconditions: finite logits (NaN/inf give unspecified ids).
 *   Errors: INVALID_ARG (T < 0; E < 1; k < 1 or k > E; null pointers with T > 0;
 *   unknown dtype or flags), UNSUPPORTED (E > 1024 or k > 32).  T == 0 is a no-op.
 */
MOE_API moe_status_t moe_topk_softmax(const void* logits, moe_dtype_t dtype, int64_t T, int32_t E, int32_t k,
                              uint32_t flags, float* topk_weights, int32_t* topk_ids, void* stream);

/*
 * Rows of the block-padded expert-grouped layout: C = T*k + E_local*(bs-1), an
 * upper bound of N_pad for every routing (each local expert pads < bs rows).
 * Returns -1 for invalid sizes.  Host-only, no CUDA call.
 */
MOE_API int64_t moe_align_capacity(int64_t T, int32_t k, int32_t E_local, int32_t block_size);

/* Blocks of the layout: ceil(C / bs), the length of expert_ids.  -1 for invalid sizes. */
MOE_API int64_t moe_align_num_blocks(int64_t T, int32_t k, int32_t E_local, int32_t block_size);

/*
 * Bytes of device workspace moe_align_permute needs for these sizes (a status
 * word, a completion ticket, per-tile expert counters and the expert totals).  Host-only.
 * The workspace must be zero-filled once before its first use (see
 * moe_workspace_init); every call leaves it ready for the next one.  The first
 * 4 bytes are the device status word that moe_read_status reads; pass the
 * workspace pointer as `device_status` to moe_gather/moe_combine to collect
 * their errors in the same word.
 */
MOE_API size_t moe_align_workspace_bytes(int64_t T, int32_t k, int32_t E_local);

/* Zero `bytes` of workspace on `stream` (cudaMemsetAsync).  Capture-safe. */
MOE_API moe_status_t moe_workspace_init(void* workspace, size_t bytes, void* stream);

/*
 * moe_align_permute -- histogram, padded prefix and stable placement of the
 * routed slots ("Upstream Reference", "File Index": moe_align_sum_kernels.cu;
 * compact scheduler note, scheduler and coverage paragraphs).
 *   topk_ids          [T, k] int32: global expert ids (any producer; duplicates
 *                     within a row are allowed).
 *   expert_map        [E_global] int32 global -> local expert, -1 = remote (not
 *                     on this rank), or NULL for the identity (then E_local must
 *                     equal E_global).  Non-negative values should be distinct.
 *   Outputs (C = moe_align_capacity, NB = moe_align_num_blocks):
 *   counts            [E_local]   local slots per expert
 *   offsets           [E_local+1] exclusive prefix of ceil(counts/bs)*bs;
 *                                 offsets[E_local] = N_pad
 *   sorted_token_ids  [C]  row -> slot id s; the slots of expert e fill rows
 *                          offsets[e] .. offsets[e]+counts[e]-1 in ascending s
 *                          (stable by expert, token, slot); every other row
 *                          (pads, and rows N_pad..C-1) holds T*k
 *   expert_ids        [NB] expert of each bs-row block; -1 from block N_pad/bs on
 *   num_tokens_post_pad [1] N_pad
 *   inv_perm          [T*k] slot -> row, -1 for a remote slot
 *   A slot whose id is outside [0, E_global), or whose mapped value is outside
 *   [-1, E_local), is treated as remote and MOE_ERR_BAD_EXPERT_ID is recorded.
 *   An all-remote rank is valid: counts 0, N_pad 0, all rows pads.
 *   Deterministic: the outputs depend only on the inputs (no atomic ordering).
 *   workspace: >= moe_align_workspace_bytes(T, k, E_local) bytes, zeroed before
 *   the first use; calls that share a workspace must not overlap on the GPU.
 *   Errors: INVALID_ARG (sizes, null pointers, E_local > E_global, identity map
 *   with E_local != E_global, T*k >= 2^30, C >= 2^31), UNSUPPORTED
 *   (E_local > 1024), WORKSPACE.  T == 0 still writes every output.
 */
MOE_API moe_status_t moe_align_permute(const int32_t* topk_ids, int64_t T, int32_t k, int32_t E_global,
                               const int32_t* expert_map, int32_t E_local, int32_t block_size,
                               int32_t* counts, int32_t* offsets, int32_t* sorted_token_ids,
                               int32_t* expert_ids, int32_t* num_tokens_post_pad, int32_t* inv_perm,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * moe_align_permute_noalloc -- moe_align_permute without a workspace argument.  The pages
 * have no counterpart of this entry point; it exists for callers that cannot allocate device
 * memory: a host framework whose custom-op interface passes only the op's own inputs and
 * outputs and does not let the op call cudaMalloc (for example because the call may run while
 * the stream is being captured, or because another component owns the device memory budget).
 *   Same arguments, outputs, ordering and errors as moe_align_permute, except:
 *   - no workspace: the completion ticket and the per-tile expert counters live in a fixed
 *     1 MiB array inside the library, one per GPU that loads it, held until the process exits;
 *   - it always runs the count + place tile kernels; sizes whose scratch would exceed that
 *     array return MOE_ERR_UNSUPPORTED before anything is enqueued.  The scratch is a 256-byte
 *     header plus 4 bytes per local expert per tile; a tile holds 2048 slots, doubled (up to
 *     8192) while there would be more than 256 tiles, and above 4096 slots at least 16 tiles'
 *     counters are kept.  With E_local = 1024, for example, up to 2 088 960 slots fit, except
 *     522 241 to 524 288 and 1 044 481 to 1 048 576 (256 tiles);
 *   - device_status: a caller device int32 that collects device-side errors, or NULL.
 *   It calls no cudaMalloc, cudaFree or other allocating routine.  The first call in each
 *   CUDA context (the device's primary context; again after a device reset, which makes a new
 *   one) looks up the array's device address (cudaGetSymbolAddress) with that device current
 *   and caches it under the context's id; make that first call before any stream capture.
 *   Each call clears the ticket
 *   with an asynchronous 4-byte memset on `stream`; the counters are rewritten before they
 *   are read.  All calls on a device share the one array and it keeps the last call's
 *   contents, so calls that overlap on the GPU (different streams, concurrent graphs) race
 *   and give wrong results: serialise them.
 */
MOE_API moe_status_t moe_align_permute_noalloc(const int32_t* topk_ids, int64_t T, int32_t k, int32_t E_global,
                                               const int32_t* expert_map, int32_t E_local, int32_t block_size,
                                               int32_t* counts, int32_t* offsets, int32_t* sorted_token_ids,
                                               int32_t* expert_ids, int32_t* num_tokens_post_pad,
                                               int32_t* inv_perm, int32_t* device_status, void* stream);

/*
 * moe_gather -- permute-gather of the activations into the expert-grouped
 * layout ("expand" of the FusedMoE pipeline, "Upstream Reference", "File Index";
 * "final permuted gather" of the compact scheduler note).
 *   hidden     [T, H] bf16.
 *   inv_perm   [T*k] int32 from moe_align_permute.
 *   permuted   [capacity, H] bf16 out: row inv_perm[s] = hidden[s / k] for every
 *              local slot s (bit copy).  Pad rows are untouched unless
 *              MOE_GATHER_ZERO_PAD, which writes +0 to every pad row below N_pad
 *              (this needs sorted_token_ids and num_tokens_post_pad; otherwise
 *              they may be NULL).  Rows >= N_pad are never written.
 *   Each hidden row is read once and written to all its local destinations.
 *   Without MOE_GATHER_HIDDEN_READY the rows are read after inv_perm, and the
 *   row of a token with no local slot is not read at all (in an expert-parallel
 *   layer, hidden may be another GPU's memory).
 *   device_status: a device int32 (e.g. the align workspace) or NULL; a row
 *   outside [-1, capacity) is skipped and MOE_ERR_BAD_ROW recorded.
 *   Errors: INVALID_ARG (sizes, null pointers, H % 8 != 0, misaligned pointers).
 */
MOE_API moe_status_t moe_gather(const void* hidden, int64_t T, int32_t H, int32_t k, const int32_t* inv_perm,
                        const int32_t* sorted_token_ids, const int32_t* num_tokens_post_pad, int64_t capacity,
                        uint32_t flags, void* permuted, int32_t* device_status, void* stream);

/*
 * moe_combine -- top-k weighted combine back to token order ("combine" of the
 * FusedMoE pipeline and the "sum" of moe_align_sum_kernels.cu, "Upstream
 * Reference", "File Index").
 *   expert_out    [capacity, H] bf16: one row per expert-grouped row.
 *   topk_weights  [T, k] fp32; inv_perm [T*k] int32 (from moe_align_permute).
 *   out           [T, H] bf16: out[t,h] = bf16_rne(acc), acc = +0.0f then, for
 *                 j = 0..k-1 with r = inv_perm[t*k+j] >= 0,
 *                 acc = fmaf(w[t,j], expert_out[r,h], acc).  Remote slots add
 *                 nothing (an expert-parallel partial sum; +0 for a token with
 *                 no local slot).
 *   device_status: as for moe_gather.
 *   Errors: INVALID_ARG (sizes, null pointers, H % 8 != 0, misaligned pointers).
 */
MOE_API moe_status_t moe_combine(const void* expert_out, const float* topk_weights, const int32_t* inv_perm, int64_t T,
                         int32_t k, int32_t H, int64_t capacity, void* out, int32_t* device_status, void* stream);

/*
 * moe_route_dispatch -- gating, align and permute-gather in one call, as three kernels (one for
 * small batches) instead of the stage calls' four or more ("Upstream Reference", "File Index": the
 * gate -> topk -> expand part of the FusedMoE pipeline).  Every output is the same as from moe_topk_softmax (flags: MOE_RENORMALIZE) then
 * moe_align_permute then moe_gather (without MOE_GATHER_ZERO_PAD), bit for bit:
 *   topk_weights [T,k], topk_ids [T,k], counts [E_local], offsets [E_local+1],
 *   sorted_token_ids [C], expert_ids [NB], num_tokens_post_pad [1], inv_perm [T*k],
 *   permuted [C, H] (rows of local slots; pad rows untouched).
 * For T > 32, T*k > 256 or E > 256: the first kernel gates tiles of tokens and counts each tile's slots
 * per local expert with their ranks inside the tile; the second turns each expert's tile counts into
 * its prefix over the tiles and its total; the third scans the padded totals into the offsets, gives
 * every slot its row and copies the hidden rows there.  Smaller batches (decode) take one kernel with one
 * CTA per slot: each CTA routes the whole batch by itself, writes its own slot's row and a share of the
 * other routing outputs, and copies the hidden row of its slot.
 *   logits [T, E] bf16/fp32 (dtype); hidden [T, H] bf16, 16-byte aligned, H % 8 == 0 and
 *   H <= 65536; expert_map and E_local as for moe_align_permute.
 *   flags: MOE_RENORMALIZE, MOE_SCORING_SIGMOID (as for moe_topk_softmax);
 *   MOE_DISPATCH_GIVEN_IDS: the routes in topk_ids [T,k] are the
 *   input (the align input of moe_align_permute), logits and topk_weights may be NULL and are
 *   not read or written; every other output is as from moe_align_permute + moe_gather.
 *   workspace: >= moe_route_dispatch_workspace_bytes(T, k, E_local) bytes, zeroed before its
 *   first use and left ready by every call; its first 4 bytes are the device status word.  Words
 *   2 and 3 are test hooks and must stay zero in normal use (moe_workspace_init zeroes them): a
 *   nonzero word 2 makes the placement kernel withhold its hidden-row loads so that its bounded wait
 *   runs out (MOE_ERR_TIMEOUT), word 3 sets that wait's limit in microseconds.
 *   Errors: as the three calls it replaces; UNSUPPORTED also for H > 65536.
 */
MOE_API size_t moe_route_dispatch_workspace_bytes(int64_t T, int32_t k, int32_t E_local);

MOE_API moe_status_t moe_route_dispatch(const void* logits, moe_dtype_t dtype, const void* hidden, int64_t T,
                                        int32_t E, int32_t k, int32_t H, uint32_t flags, const int32_t* expert_map,
                                        int32_t E_local, int32_t block_size, float* topk_weights, int32_t* topk_ids,
                                        int32_t* counts, int32_t* offsets, int32_t* sorted_token_ids,
                                        int32_t* expert_ids, int32_t* num_tokens_post_pad, int32_t* inv_perm,
                                        void* permuted, void* workspace, size_t workspace_bytes, void* stream);

/*
 * moe_reduce_partials -- the exchange after an expert-parallel combine: the sum of
 * the ranks' partial combines ("b70-optimization-lab: 2026-07-16 MTP1 M=2 compact
 * scheduler closure note", scheduler paragraph: each rank keeps the slots of its own
 * experts through expert_map, so its moe_combine is a partial sum over its local
 * slots; the note leaves the collective that sums them out).
 *   partials    HOST array of n_partials DEVICE pointers, the partials in rank order,
 *               each [rows, H] bf16, 16-byte aligned.  A pointer may address another
 *               GPU's memory (peer access enabled): it is read with plain 16-byte loads.
 *               The array itself is read during the call only.
 *   n_partials  1..16.
 *   out         [rows, H] bf16 out: each element is the fp32 sum of the partials'
 *               elements in ascending rank order from +0, rounded once to bf16
 *               (round-to-nearest-even).  out may be one of the partials (every
 *               element is read before it is written).
 *   For a reduce-scatter, rank r's moe_combine writes owner o's token range of its
 *   partial into owner o's receive buffer (`out` pointing into the owner's memory, with
 *   topk_weights and inv_perm advanced to the range's first token); once every rank has
 *   written (the caller's barrier), owner o calls moe_reduce_partials on its buffers.
 *   Errors: INVALID_ARG (rows < 0, H % 8 != 0, rows * H beyond 2^47, null or misaligned
 *   pointers), UNSUPPORTED (n_partials > 16).
 */
MOE_API moe_status_t moe_reduce_partials(const void* const* partials, int32_t n_partials, int64_t rows, int32_t H,
                                         void* out, void* stream);

/*
 * Read the device status word (first 4 bytes of an align workspace, or any
 * device int32 used as device_status), reset it to MOE_OK, and return the
 * value in *device_status.  Synchronises `stream`.  Not capturable.
 */
MOE_API moe_status_t moe_read_status(int32_t* device_status_word, void* stream, moe_status_t* device_status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_ROUTE_H_ */

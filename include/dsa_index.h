/*
 * dsa_index.h — C ABI of libdsaidx, a B200 (sm_100a) library for the
 * DeepSeek Sparse Attention (DSA) lightning indexer and two scan-reducing
 * variants of it.
 *
 * What is computed.  For query t of a sequence (H heads of dimension d, a
 * weight per head) and key s of the same sequence (one key per token, shared
 * by every head) the indexer score is
 *
 *        I[t,s] = sum_h  w[t,h] * max(0, q[t,h] . k[s])
 *
 * and the indexer keeps, for every query, the k keys with the highest score
 * among its causal prefix.  The pages this library follows describe the
 * indexer in words only ("Multi-layer Indexer: overlapping selection and
 * attention in DeepSeek Sparse Attention", abstract: the indexer scores the
 * whole cache and keeps the k = 2048 best tokens; "PIVOT: Efficient
 * Query-Group Indexing for Token-Level Sparse Attention", abstract: each
 * query scores every preceding token).  The formula is DeepSeek-V3.2's.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  Data types and layouts (row-major, densely packed, device memory):
 *    Q  [n_q, H, d]  bf16 (passed as const void*), rows 16-byte aligned
 *    K  [n_k, d]     bf16, rows 16-byte aligned
 *    W  [n_q, H]     fp32
 *  Sequences.  A batch holds B sequences.  Sequence b owns query rows
 *  [q_offsets[b], q_offsets[b+1]) and key rows [k_offsets[b],
 *  k_offsets[b+1]).  q_pos[t] is query t's position inside its sequence.
 *  Causality.  Query t may select key s (a sequence-local index) when
 *  s <= q_pos[t] and s < L_b (the key count of its sequence): the query's
 *  own token is part of its prefix.  A negative position leaves the row
 *  empty.
 *  Ranking.  Higher score first; equal scores go to the lower key index.
 *  A score of -0 ranks as +0.
 *  Output rows.  Every index row holds min(k, #eligible) sequence-local key
 *  indices in ASCENDING index order, then -1 padding up to k.  Optional
 *  score outputs hold the fp32 score of each returned index (NaN padding).
 *  Supported shapes.  H a power of two in 1..64; d in {32, 64, 128};
 *  1 <= k <= 16384; a ranked row (a sequence's keys for the dense top-k and
 *  PIVOT's proxy scan, its middle blocks for HISA's block filter) of at most
 *  774,144 columns (for k below 16,128; a little more above): the selection
 *  keeps two bitmaps of the row's columns in shared memory.  Otherwise
 *  DSA_ERR_UNSUPPORTED.
 *  Ownership.  The caller owns every buffer: inputs, outputs and the
 *  workspace.  The library allocates no device memory, never synchronises
 *  the stream (dsa_device_check and dsa_profile_read excepted) and keeps no
 *  per-call state.
 *  Workspace.  Every call that takes `ws` needs at least the bytes its
 *  *_workspace function returns for the same arguments, 256-byte aligned.
 *  Its first 256 bytes hold a device status word: kernels that detect a
 *  problem (a bounded wait that ran out) record it there and return early;
 *  dsa_device_check reads it.  Calls overlapping on the GPU need distinct
 *  workspaces.
 *  Streams.  `stream` is a cudaStream_t (NULL = legacy default stream).  All
 *  work is enqueued on it; results are ready when the stream reaches them.
 *  Errors.  Argument checks run on the host before anything is enqueued and
 *  return DSA_ERR_INVALID_ARG / DSA_ERR_UNSUPPORTED / DSA_ERR_WORKSPACE with
 *  nothing launched.  A failed launch returns DSA_ERR_CUDA.  Faults that
 *  happen later on the device surface at the caller's next synchronisation.
 *  Non-finite inputs give undefined rankings.
 *  Thread safety.  Entry points may be called from several host threads
 *  at once given distinct workspaces.
 */
#ifndef DSA_INDEX_H
#define DSA_INDEX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dsa_status {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad offsets, misalignment */
    DSA_ERR_UNSUPPORTED = 2,   /* shape outside the supported set */
    DSA_ERR_WORKSPACE = 3,     /* workspace missing, too small or misaligned */
    DSA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    DSA_ERR_DEVICE_CHECK = 5   /* a kernel recorded an error in the workspace status word */
} dsa_status;

/* A ragged batch of sequences.  The device arrays are read by the kernels;
 * the host copies (same values) size grids and workspaces without a
 * device-to-host copy.  All pointers stay owned by the caller. */
typedef struct dsa_batch {
    int32_t num_seqs;              /* B >= 1 */
    int32_t num_heads;             /* H */
    int32_t head_dim;              /* d */
    int32_t num_queries;           /* n_q = q_offsets[B] (may be 0) */
    int32_t num_keys;              /* n_k = k_offsets[B] */
    const int32_t* q_offsets;      /* device [B+1], non-decreasing, q_offsets[0] = 0 */
    const int32_t* k_offsets;      /* device [B+1], non-decreasing, k_offsets[0] = 0 */
    const int32_t* q_pos;          /* device [n_q] */
    const int32_t* q_offsets_host; /* host   [B+1] */
    const int32_t* k_offsets_host; /* host   [B+1] */
} dsa_batch;

/* Human-readable name of a status code (static storage). */
const char* dsa_status_string(dsa_status status);

/* Library version, major*10000 + minor*100 + patch. */
int32_t dsa_version(void);

/* --------------------------------------------------------------------
 * Dense indexer scores (debug / reference view of the contraction).
 * S [n_q, ld_s] fp32: S[t][s] = I[t,s] for eligible s, -inf for every other
 * s < ld_s.  ld_s >= the longest sequence's key count.  The full score matrix
 * is written, so this call is for inspection, not the hot path.
 * Source: the indexer score of the MLI and PIVOT abstracts.
 */
size_t dsa_index_scores_workspace(const dsa_batch* batch);
dsa_status dsa_index_scores(const dsa_batch* batch, const void* Q, const void* K, const float* W,
                            float* S, int64_t ld_s, void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------------
 * Dense indexer top-k: for every query, the k best eligible keys.
 * idx [n_q, k] int32; scores [n_q, k] fp32 or NULL.
 * Source: MLI abstract (score the whole cache, keep k = 2048); PIVOT
 * abstract (every preceding token is scored, O(L^2) per layer in prefill).
 * Prefill (one query per position) and batched decode (a few MTP queries
 * per sequence at its end) are the same call with different q_pos.
 */
size_t dsa_index_topk_workspace(const dsa_batch* batch, int32_t k);
dsa_status dsa_index_topk(const dsa_batch* batch, const void* Q, const void* K, const float* W,
                          int32_t k, int32_t* idx, float* scores, void* ws, size_t ws_bytes,
                          void* stream);

/* --------------------------------------------------------------------
 * Cross-layer index reuse: the selections of n_layers consecutive layers
 * from fewer indexer runs.  Two schedules from the pages, combinable:
 *  - retain_every = r (IndexCache, as the MLI abstract and the related-paper
 *    list of the PIVOT page describe it: a few "full" layers run their own
 *    indexer, the "shared" layers reuse the nearest full layer's top-k; a keep
 *    ratio of 1/r): layer l's indexer runs only when l % r == 0; every other
 *    layer reuses the selection of the nearest full layer below it.
 *  - lag = 1 ("Multi-layer Indexer: overlapping selection and attention in
 *    DeepSeek Sparse Attention", abstract): layer l attends over the selection
 *    made for layer l - 1, so layer l's own indexer can run beside layer
 *    l - 1's attention; layer 0 uses its own.  lag = 0: each layer uses the
 *    selection of its own (nearest indexed) layer.
 * dsa_index_layers_source(l, r, lag) is the layer whose indexer produces
 * layer l's selection: r * floor((lag && l > 0 ? l - 1 : l) / r); -1 for a
 * negative l, r < 1 or lag not 0/1.  Host-only.
 * dsa_index_layers: Q, K, W and idx are HOST arrays of n_layers DEVICE
 * pointers (layer l's inputs, laid out as for dsa_index_topk; every layer
 * shares `batch`).  idx[l] [n_q, k] receives layer l's selection.  Each
 * indexer run that some layer consumes is made by dsa_index_topk on
 * `side_stream` (after the work already on `stream`), written into its first
 * consumer's rows and copied to the others; runs nobody consumes are skipped.
 * ready_events: NULL, or a HOST array of n_layers cudaEvent_t (created by the
 * caller): event l is recorded on side_stream once idx[l] is complete, so the
 * caller's work for layer l waits for that alone.  With NULL, `stream` waits
 * for every selection before its later work.  The workspace is
 * dsa_index_topk's (dsa_index_layers_workspace), reused by the runs in turn.
 * side_stream must differ from stream.
 */
int32_t dsa_index_layers_source(int32_t layer, int32_t retain_every, int32_t lag);
size_t dsa_index_layers_workspace(const dsa_batch* batch, int32_t k);
dsa_status dsa_index_layers(const dsa_batch* batch, int32_t n_layers, const void* const* Q, const void* const* K,
                            const float* const* W, int32_t k, int32_t retain_every, int32_t lag, int32_t* const* idx,
                            void* const* ready_events, void* ws, size_t ws_bytes, void* stream, void* side_stream);

/* --------------------------------------------------------------------
 * Dense top-k from host memory (no counterpart in the pages; the same
 * computation as dsa_index_topk for inputs that live in host memory).
 * Q, K, W, q_pos_host and idx are HOST pointers (page-locked for the copies
 * to overlap; pageable memory works but serialises); batch->q_offsets_host
 * and k_offsets_host are used and the batch's device pointer fields are
 * ignored.  The rows are cut into chunks (about eight, of at least 2048
 * rows, within dsa_index_topk's score buffer) taken in order of decreasing
 * work (eligible pairs, counted on the host from q_pos_host): while one
 * chunk is scored and selected on `stream`, the next two chunks' queries are
 * copied in on `in_stream` and earlier chunks' indices copied out on
 * `out_stream` (K, W and q_pos are copied once, first).  in_stream and
 * out_stream must differ from `stream` (they may be the same stream, which
 * serialises the two directions).  Returns after enqueueing; idx is
 * complete when `stream` has passed the call's work.  The workspace
 * (dsa_index_topk_host_workspace bytes) holds dsa_index_topk's workspace
 * followed by device copies of K, W, q_pos, the offsets and three chunks of
 * queries and of indices.  The status word is at the workspace start as
 * for every call.
 */
size_t dsa_index_topk_host_workspace(const dsa_batch* batch, int32_t k);
dsa_status dsa_index_topk_host(const dsa_batch* batch, const int32_t* q_pos_host, const void* Q, const void* K,
                               const float* W, int32_t k, int32_t* idx, void* ws, size_t ws_bytes,
                               void* stream, void* in_stream, void* out_stream);

/* --------------------------------------------------------------------
 * PIVOT group-proxy indexing ("PIVOT: Efficient Query-Group Indexing for
 * Token-Level Sparse Attention", abstract).
 * Groups: inside each sequence, consecutive runs of `group` query rows (the
 * last run may be shorter); in decode pass group >= the MTP query count so
 * that a group is one MTP step.  Groups are numbered in sequence order;
 * pivot_num_groups returns their count.
 * Proxy: q_bar = bf16(mean of the group's q, rounded to nearest even),
 * w_bar = mean of the group's w.  The proxy scans its sequence's keys
 * s <= max q_pos of the group and keeps the n_cand best (the candidate set).
 * mode 0 (Reuse):  query t takes the k best candidates by proxy score among
 *                  candidates s <= q_pos[t].
 * mode 1 (Refine): query t scores the candidates s <= q_pos[t] with its own
 *                  q and w and takes its own top k.
 * idx [n_q, k] int32 (rows in query order); cand [n_groups, n_cand] int32 or
 * NULL (ascending, -1 padded).  Requires k <= n_cand <= 16384, 1 <= group <= 64.
 */
int32_t pivot_num_groups(const dsa_batch* batch, int32_t group);
size_t pivot_group_index_workspace(const dsa_batch* batch, int32_t k, int32_t group,
                                   int32_t n_cand, int32_t mode);
dsa_status pivot_group_index(const dsa_batch* batch, const void* Q, const void* K, const float* W,
                             int32_t k, int32_t group, int32_t n_cand, int32_t mode, int32_t* idx,
                             int32_t* cand, void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------------
 * Refine on supplied candidates: the second stage of PIVOT Refine over the
 * caller's candidate lists instead of a proxy scan - a selection made once
 * and refined by others, as the followers of an anchor layer ("LatentIndex",
 * abstract) or a group's token bank ("ADIndex: Layer-Adaptive Sparse
 * Attention Indexing via Group-Level Distillation", abstract).
 * Groups as in pivot_group_index.  cand [n_groups, n_cand] int32 (device,
 * read only): group g's candidates, sequence-local key indices, strictly
 * ascending, then -1 padding.  Query t scores the candidates s <= q_pos[t]
 * of its group with its own q and w and takes its top k; idx as in
 * pivot_group_index.  A list that is not ascending, holds a key outside its
 * sequence or has a key after its padding is used up to its first bad entry
 * and reported through the workspace status word (code 2, read with
 * dsa_device_check).  Requires k <= n_cand <= 16384, 1 <= group <= 64.
 */
size_t pivot_refine_candidates_workspace(const dsa_batch* batch, int32_t k, int32_t group, int32_t n_cand);
dsa_status pivot_refine_candidates(const dsa_batch* batch, const void* Q, const void* K, const float* W,
                                   int32_t k, int32_t group, int32_t n_cand, const int32_t* cand,
                                   int32_t* idx, void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------------
 * HISA hierarchical indexing ("HISA: Efficient Hierarchical Indexing for
 * Fine-Grained Sparse Attention", abstract).
 * hisa_pool_keys: pooled [n_blocks, d] fp32, the mean of the keys of each
 * block of `block` tokens (the last block of a sequence may be partial);
 * blocks of all sequences stacked in order, hisa_num_blocks of them.
 * hisa_index: for query t, with last = q_pos[t] / block (clamped to the
 * sequence), the blocks strictly between block 0 and `last` are scored with
 * the indexer formula against their pooled key; block 0, block `last` and the
 * `keep` best middle blocks are kept; the indexer then ranks every eligible
 * token of the kept blocks and returns its top k.  Block scores take the fp32
 * pooled key exactly (as the sum of three bf16 parts) with fp32 accumulation.
 * The workspace includes a bf16 copy of the pooled keys (6 bytes per element)
 * when every stage runs in one launch (at most 480 sequences, rows of at most
 * 16,384 blocks and kept tokens).
 * idx [n_q, k]; kept [n_q, keep+2] int32 or NULL (ascending, -1 padded).
 * Requires block in {64, 128, 256}, 1 <= keep <= 256.
 */
int64_t hisa_num_blocks(const dsa_batch* batch, int32_t block);
dsa_status hisa_pool_keys(const dsa_batch* batch, const void* K, int32_t block, float* pooled,
                          void* stream);
size_t hisa_index_workspace(const dsa_batch* batch, int32_t k, int32_t block, int32_t keep);
dsa_status hisa_index(const dsa_batch* batch, const void* Q, const void* K, const float* W,
                      const float* pooled, int32_t k, int32_t block, int32_t keep, int32_t* idx,
                      int32_t* kept, void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------------
 * Reads the workspace status word written by the kernels of earlier calls
 * on `stream` (synchronises the stream).  Returns DSA_OK when no kernel
 * recorded a problem, else DSA_ERR_DEVICE_CHECK and, if `detail` is not
 * NULL, the recorded code (see the kernels' documentation).  Clears it.
 */
dsa_status dsa_device_check(void* ws, void* stream, uint32_t* detail);

/* --------------------------------------------------------------------
 * Self-test of the bounded waits (no counterpart in the pages; a check of
 * this library's failure reporting).  Every wait of the library's kernels on
 * an mbarrier gives up after a time limit (1 s), records code 1 (wait ran
 * out) in the workspace status word and lets the kernel finish.  This call
 * launches one CTA that waits, through the same wait routine, on a barrier
 * nothing ever completes, with a limit of `limit_us` microseconds
 * (1 .. 1000000): the wait runs out, the kernel records code 1 and returns,
 * and the context stays usable.  A later dsa_device_check on the same stream
 * reports DSA_ERR_DEVICE_CHECK with detail 1.  `ws` needs 256 bytes; the
 * call clears its status word first.  DSA_ERR_INVALID_ARG for a null or
 * misaligned `ws`, a short `ws_bytes` or a limit outside the range.
 */
dsa_status dsa_selftest_wait_timeout(uint32_t limit_us, void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------------
 * Allocation-free dense top-k (no counterpart in the pages; a convenience of
 * this library).  Same computation, arguments and outputs as dsa_index_topk,
 * but the workspace is a device array inside the library, for callers that
 * cannot call cudaMalloc (for example a custom-op callback of an inference
 * runtime that is given no allocator and must not allocate while it runs).
 *  - Capacity: dsa_index_topk_static_capacity() bytes (8 MiB), held by every
 *    GPU that loads the library until the process exits.  A batch whose
 *    dsa_index_topk_workspace exceeds it is rejected with DSA_ERR_WORKSPACE
 *    before anything is launched.
 *  - Every call looks up the array's device address in the current
 *    device's context (cudaGetSymbolAddress, which allocates nothing), so a
 *    context destroyed and made again (cudaDeviceReset) is followed.  The
 *    first lookup on a device may load the library's device code: make the
 *    first call on each device before any stream capture.
 *  - Every call on a device shares the one array: calls that overlap on the
 *    GPU (different streams, or different host threads) race and corrupt each
 *    other's results.  Serialise them.
 *  - Allocates nothing (no cudaMalloc, cudaFree or allocating library call).
 */
size_t dsa_index_topk_static_capacity(void);
dsa_status dsa_index_topk_static(const dsa_batch* batch, const void* Q, const void* K, const float* W,
                                 int32_t k, int32_t* idx, float* scores, void* stream);

/* --------------------------------------------------------------------
 * Launch accounting and kernel timing, for benchmarks (not part of the
 * indexer; no counterpart on the pages).  The only process-wide state of
 * the library.
 * dsa_launch_count: kernels launched by this library since load.
 * dsa_profile_enable(1): from then on every launch is bracketed by two CUDA
 * events recorded on its own stream.  dsa_profile_read synchronises those
 * events, adds up per kernel kind (index 0 .. n-1, names from
 * dsa_profile_kind_name) the elapsed milliseconds and launch counts into
 * ms[] / launches[] (each `cap` long, either may be NULL), forgets them, and
 * returns the number of kinds (or -1 if an event failed).
 */
void dsa_profile_enable(int32_t on);
uint64_t dsa_launch_count(void);
const char* dsa_profile_kind_name(int32_t kind);
int32_t dsa_profile_read(float* ms, int32_t* launches, int32_t cap);

#ifdef __cplusplus
}
#endif

#endif /* DSA_INDEX_H */

/*
 * dhs.h - C ABI of the B200 dynamic hashed embedding engine (libdhs.so).
 *
 * One hot path, on one GPU: a two-level dynamic hash table (an IDMap from a
 * feature id to a row offset, plus chunked EmbeddingBlocks that hold each
 * row's parameters and optimizer state and grow by appending blocks), with a
 * lookup-or-insert + sum-pooling forward and a coalesced sparse-gradient +
 * fused row-optimizer backward.
 *
 * Sources of the operations (page title, then section):
 *   [RecIS]  "RecIS: Alibaba's open-source unified training framework for
 *            recommender systems" (pomoai.com hub page), section on the
 *            Embedding Engine: IDMap (id -> offset) as the first level,
 *            EmbeddingBlocks (parameters and optimizer state, contiguous,
 *            sharded, growing without reallocation) as the second; merging
 *            tables with the same attributes; and the code-layout section:
 *            fused sparse-gradient update kernel with fewer atomics,
 *            vectorised embedding lookup.
 *   [BG]     "Alibaba RecIS: background and difficulties of search/ads/
 *            recommendation training" (muyuuuu.github.io), nn.Embedding
 *            section: a lookup reads one row, the backward updates only that
 *            row; worked SGD example with a 10 x 4 table.
 *   [DLRM-P] "DLRM model: core value and industrial deployment" (mokono.cn),
 *            section 2.1: nn.EmbeddingBag(mode="sum") for variable-length
 *            inputs with sparse gradients.
 *   [DLRM-E] "DLRM: Meta splits industrial recommendation into 4 standard
 *            blocks" (estelledc.github.io), module 2 (one table per
 *            categorical field) and pitfall 4 (sparse optimizer: only the
 *            touched rows are updated).
 *
 * Conventions for every call:
 *   - Pointers named d_* are DEVICE pointers on the table's device; pointers
 *     named h_* are HOST pointers.  The caller owns every buffer it passes;
 *     the library owns the table (IDMap, blocks, workspace).
 *   - Calls taking a stream are asynchronous and ordered on that stream
 *     (NULL = the legacy default stream).  A table is used by one host thread
 *     at a time, and its calls must be ordered (one stream, or the caller's
 *     own events).
 *   - Keys are int64 >= 0; with merged tables key = table_id << 48 | id
 *     (dhs_pack_keys).  -1 is reserved.
 *   - Argument errors are returned at once and nothing is launched.  Errors
 *     found by a kernel (a negative key, a key missing in the backward, a
 *     full table) are latched in a device word; the call's own work goes on
 *     for the valid inputs, and the first latched error is returned by the
 *     next ht_sync / ht_size / ht_export.
 *   - Floating point: fp32 storage; forward sums in fp32 in bag order;
 *     backward gradient sums in fp64, rounded once to fp32; optimizer
 *     arithmetic in fp32, each operation rounded (no contraction).
 */
#ifndef DHS_H_
#define DHS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* dhs_stream;

typedef struct dhs_table dhs_table; /* opaque, library-owned */

typedef enum {
  DHS_OK = 0,
  DHS_ERR_INVALID_ARG = 1, /* bad argument, negative key, malformed bag offsets */
  DHS_ERR_OOM = 2,         /* device allocation failed */
  DHS_ERR_CUDA = 3,        /* a CUDA runtime call failed */
  DHS_ERR_TABLE_FULL = 4,  /* row limit (max_rows) or IDMap probe bound reached */
  DHS_ERR_NOT_FOUND = 5,   /* backward saw a key that is not in the table */
  DHS_ERR_UNSUPPORTED = 6, /* configuration the library does not handle */
  DHS_ERR_INTERNAL = 7     /* a bounded device-side wait gave up (results undefined) */
} dhs_status;

typedef enum {
  DHS_SGD = 0,             /* w -= lr*g                                         */
  DHS_ADAGRAD = 1,         /* per-element G += g*g; w -= lr*g/(sqrt(G)+eps)     */
  DHS_ADAM = 2,            /* lazy Adam: m, v per element beside the row        */
  DHS_ADAGRAD_ROWWISE = 3  /* one accumulator per row: G += mean(g^2)           */
} dhs_optimizer;

/* EmbeddingBag pooling ([DLRM-P] 2.1, nn.EmbeddingBag): the sum of a bag's
 * rows (optionally weighted per id), or their mean. */
typedef enum {
  DHS_POOL_SUM = 0,
  DHS_POOL_MEAN = 1,
  /* Backward only: mean pooling carried to a key's owner by the sharded
   * engine, each id its own bag: d_per_sample_weights holds the length of
   * the id's original bag, and the id's gradient row is divided by it (in
   * fp64, as DHS_POOL_MEAN does). */
  DHS_POOL_DIVIDE = 2
} dhs_pool_mode;

typedef struct {
  float eps;   /* default 1e-8 */
  float beta1; /* Adam, default 0.9 */
  float beta2; /* Adam, default 0.999 */
} dhs_opt_params;

/* Optional device allocator (e.g. a framework's caching allocator).  alloc
 * returns device memory usable on `stream` or NULL; free releases a block
 * returned by alloc once the work on `stream` that uses it is done.  With
 * NULL the library uses cudaMallocAsync / cudaFreeAsync on the call's stream. */
typedef struct {
  void* (*alloc)(size_t bytes, dhs_stream stream, void* ctx);
  void (*free)(void* ptr, size_t bytes, dhs_stream stream, void* ctx);
  void* ctx;
} dhs_allocator;

/* Human-readable name of a status code (static string). */
const char* dhs_status_str(dhs_status s);

/* key[i] = table_ids[i] << 48 | ids[i]  ([RecIS] Embedding Engine: tables with
 * the same attributes merged into one map).  An entry with table_id outside
 * [0, 2^15) or id outside [0, 2^48) gives key -1, which a table call then
 * reports as DHS_ERR_INVALID_ARG.  d_table_ids int32[n], d_ids int64[n],
 * d_keys_out int64[n]; n = 0 is a no-op. */
dhs_status dhs_pack_keys(const int32_t* d_table_ids, const int64_t* d_ids, int64_t n,
                         int64_t* d_keys_out, dhs_stream stream);

/* Create an empty table on the current CUDA device ([RecIS] Embedding
 * Engine).  dim: embedding width, a multiple of 4 in [4, 512].  opt: the
 * optimizer whose state lives beside each row.  block_rows: rows per
 * EmbeddingBlock, a power of two (0 = 2^20).  max_rows: row limit (0 = 2^31;
 * at most 2^32 - 2).  params / alloc may be NULL (defaults).  The row stride
 * is dim * (1 + s) floats, s = 0 (SGD), 1 (Adagrad), 2 (Adam), or dim + 1
 * for row-wise Adagrad.  On success *out is a new handle. */
dhs_status ht_create(int32_t dim, dhs_optimizer opt, int64_t block_rows, int64_t max_rows,
                     const dhs_opt_params* params, const dhs_allocator* alloc,
                     dhs_table** out);

/* Storage type of the weights ([DLRM-P] 4.2: embedding matrices stored in
 * 16-bit floats to halve their bytes); the optimizer state is fp32 either way. */
typedef enum {
  DHS_ROWS_F32 = 0,
  DHS_ROWS_BF16 = 1  /* dim a multiple of 8 in [32, 512] */
} dhs_row_dtype;

/* ht_create with a weight storage type.  DHS_ROWS_BF16: each stored weight
 * (the initial row and every optimizer step's result) is rounded to the
 * nearest bf16 value, ties to even; the forward sums the stored values in
 * fp32; the optimizer computes in fp32 and rounds once on store; the state
 * stays fp32.  A bf16 row holds dim bf16 weights then the state (dim / 2 +
 * state floats, 16-byte aligned).  bf16 with dim not a multiple of 8 or below
 * 32 returns DHS_ERR_UNSUPPORTED.  ht_get_rows and ht_export return bf16
 * weights widened to fp32, so their rows have dim + state floats for both
 * types (ht_row_stride). */
dhs_status ht_create_ex(int32_t dim, dhs_optimizer opt, dhs_row_dtype weights, int64_t block_rows,
                        int64_t max_rows, const dhs_opt_params* params, const dhs_allocator* alloc,
                        dhs_table** out);

/* Wait for the table's work and release everything it owns.  NULL is a no-op. */
dhs_status ht_destroy(dhs_table* t);

/* Reserve capacity for n_keys keys now: the IDMap is grown so that it holds
 * them without rehashing, and EmbeddingBlocks covering n_keys rows (at most
 * max_rows) are appended.  No key or row is added; existing rows are
 * untouched.  Lets a caller keep allocation and rehash work out of its
 * training steps. */
dhs_status ht_reserve(dhs_table* t, int64_t n_keys, dhs_stream stream);

/* Lookup-or-insert ([RecIS] IDMap: id -> offset; [BG] row lookup).
 * d_offsets_out[i] = row offset of d_keys[i].  A key seen for the first time
 * gets the next free row; new keys of one call are numbered in the order of
 * their first position in d_keys, starting at the row count before the call,
 * and their rows are initialised from splitmix64(key) (values in
 * [-0.05, 0.05), optimizer state 0).  Rows never move.  A negative key gives
 * offset -1 and latches DHS_ERR_INVALID_ARG. */
dhs_status ht_lookup_or_insert(dhs_table* t, const int64_t* d_keys, int64_t n,
                               int64_t* d_offsets_out, dhs_stream stream);

/* Read-only lookup (no insert): offset, or -1 for an absent or negative key
 * (or one not admitted yet). */
dhs_status ht_lookup(dhs_table* t, const int64_t* d_keys, int64_t n, int64_t* d_offsets_out,
                     dhs_stream stream);

/* Forward ([DLRM-P] 2.1 EmbeddingBag sum; [BG] row lookup; [RecIS] vectorised
 * lookup): lookup-or-insert of every key, then
 *   d_pooled_out[b, :] = sum of rows of d_keys[d_bag_offsets[b] ..
 *                        d_bag_offsets[b+1]) in that order, fp32.
 * d_keys int64[n_keys]; d_bag_offsets int64[n_bags + 1], non-decreasing,
 * [0] = 0, [n_bags] = n_keys (checked on the device); d_pooled_out
 * float[n_bags, dim] row-major, 16-byte aligned.  An empty bag gives a zero
 * row.  New keys get rows exactly as in ht_lookup_or_insert. */
dhs_status embbag_forward(dhs_table* t, const int64_t* d_keys, int64_t n_keys,
                          const int64_t* d_bag_offsets, int64_t n_bags, float* d_pooled_out,
                          dhs_stream stream);

/* Backward + update ([RecIS] fused sparse-gradient update with fewer
 * atomics; [DLRM-E] pitfall 4 sparse optimizer; [BG] only touched rows change).
 * For each distinct key k of d_keys:
 *   g_k = sum over the positions i holding k of d_grad[bag(i), :]
 * (fp64 sum, rounded once), then one step of the table's optimizer on row k
 * with learning rate lr.  Rows not in d_keys are not read or written.  The
 * Adam step count advances by one per call.  Keys must be in the table
 * (missing ones are skipped and latch DHS_ERR_NOT_FOUND).
 * d_grad float[n_bags, dim] row-major, 16-byte aligned (rows are copied in
 * 16-byte pieces); the other arguments as in embbag_forward.
 * Performance note: when the table's last insert call was a forward whose
 * bags averaged at least 4 ids, over as many positions as this call, the
 * rows that forward found are reused at every position holding the same key
 * (other positions are looked up); the result does not depend on it. */
dhs_status embbag_backward_update(dhs_table* t, const int64_t* d_keys, int64_t n_keys,
                                  const int64_t* d_bag_offsets, int64_t n_bags,
                                  const float* d_grad, float lr, dhs_stream stream);

/* embbag_forward with EmbeddingBag's other forms ([DLRM-P] 2.1: the module
 * nn.EmbeddingBag, whose definition includes mode="mean" and per-sample
 * weights).  d_per_sample_weights: NULL, or float[n_keys] (device), one
 * weight per id, allowed with DHS_POOL_SUM only:
 *   DHS_POOL_SUM   pooled[b] = sum of fl(w_i * row(key_i)) in bag order
 *                  (no weights: the plain sum of embbag_forward);
 *   DHS_POOL_MEAN  pooled[b] = fl(sum of rows / (float)len_b), one rounded
 *                  division of the fp32 in-order sum; an empty bag gives 0.
 * Mean pooling with weights, or an unknown mode, returns
 * DHS_ERR_INVALID_ARG at once.  Everything else as in embbag_forward. */
dhs_status embbag_forward_ex(dhs_table* t, const int64_t* d_keys, int64_t n_keys,
                             const int64_t* d_bag_offsets, int64_t n_bags, const float* d_per_sample_weights,
                             dhs_pool_mode mode, float* d_pooled_out, dhs_stream stream);

/* embbag_backward_update for the forms of embbag_forward_ex: the pooled
 * output's gradient reaches occurrence i scaled by w_i (per-sample weights)
 * or by 1 / len(bag of i) (mean pooling), so
 *   g_k = sum over the positions i holding k of f_i * d_grad[bag(i), :],
 * with f_i * grad formed and summed in fp64 and rounded once to fp32, then
 * one optimizer step as in embbag_backward_update.  The weights and mode must
 * be those of the forward.  Same argument rules as embbag_forward_ex. */
dhs_status embbag_backward_update_ex(dhs_table* t, const int64_t* d_keys, int64_t n_keys,
                                     const int64_t* d_bag_offsets, int64_t n_bags,
                                     const float* d_per_sample_weights, dhs_pool_mode mode,
                                     const float* d_grad, float lr, dhs_stream stream);

/* Allocation-free variant of embbag_backward_update (the pages have no
 * counterpart: it exists for callers that cannot allocate device memory
 * during a step, e.g. a runtime that forbids cudaMalloc once its training
 * loop runs, or one that gives this library only the buffers it owns).
 * Same arguments, same result as embbag_backward_update; the sort and
 * segment-reduce scratch is one fixed file-scope device array (about 12 MB,
 * held by every GPU that loads this library until the process exits)
 * instead of the table's growable workspace, and no cudaMalloc, cudaFree or
 * allocating library routine is called.
 * Limits: n_keys <= DHS_NOALLOC_MAX_KEYS and a table dim <= 128; larger calls
 * return DHS_ERR_INVALID_ARG and do nothing.
 * The first call on a device looks the array's address up
 * (cudaGetSymbolAddress) and caches it: make that first call before any
 * stream capture.  All calls share the one array, so calls whose work
 * overlaps on the GPU (different streams, or different tables on the same
 * device without ordering) race; order them. */
#define DHS_NOALLOC_MAX_KEYS 131072
dhs_status embbag_backward_update_noalloc(dhs_table* t, const int64_t* d_keys, int64_t n_keys,
                                          const int64_t* d_bag_offsets, int64_t n_bags,
                                          const float* d_grad, float lr, dhs_stream stream);

/* Feature admission and eviction ([RecIS] code-layout section: the
 * HashtableHook admission / eviction strategy of the embedding engine; the
 * pages give only its name, so the behaviour below is this library's
 * reading).  Call on a new table, before its first insert call, at most once.
 *   admit_threshold: a key gets a row in the first insert call (forward or
 *     lookup-or-insert) in which its occurrences over all such calls, this
 *     call's included, reach the threshold (0 or 1: at first sight).  Until
 *     then it pools as a zero row, lookups give -1, its gradients are skipped
 *     (not an error) and its count is kept.  Keys admitted by one call get
 *     rows in the order of their first position in it.
 *   track_access: every insert call is one step and stamps the keys that
 *     occur in it; needed by ht_evict.
 * With either set, forward calls always take the split forward (probe,
 * assignment, gather).  Returns DHS_ERR_INVALID_ARG on a used table. */
dhs_status ht_set_hooks(dhs_table* t, int64_t admit_threshold, int track_access);

/* Evict every key (with or without a row) whose last occurrence is more than
 * max_idle insert calls back (stamp < calls so far - max_idle): its IDMap
 * slot becomes a tombstone (skipped by probes, dropped by the next rehash)
 * and its row becomes free.  Later new keys take the free rows in ascending
 * order before rows are appended; a reused row starts from its new key's
 * initial values and zero state.  An evicted key that occurs again is a new
 * key.  Synchronous: waits for the stream, then *n_freed = rows freed.
 * Needs track_access (else DHS_ERR_INVALID_ARG).  ht_size still counts
 * every row ever appended; ht_export gives key -1 for a free row. */
dhs_status ht_evict(dhs_table* t, int64_t max_idle, int64_t* n_freed, dhs_stream stream);

/* *n_live = rows held by keys (appended rows minus free ones).  Synchronises
 * like ht_sync and returns its status. */
dhs_status ht_live_rows(dhs_table* t, int64_t* n_live);

/* Copy the full rows (dim weights, then the state) of the given keys into
 * d_rows_out float[n, ht_row_stride(t)]; an absent key gives a NaN row. */
dhs_status ht_get_rows(dhs_table* t, const int64_t* d_keys, int64_t n, float* d_rows_out,
                       dhs_stream stream);

/* Floats per row as ht_get_rows / ht_export return it (dim weights as fp32,
 * then the optimizer state), or -1 for a NULL handle. */
int64_t ht_row_stride(const dhs_table* t);

/* Wait for all the table's work; return the first latched device error (and
 * clear it), else DHS_OK. */
dhs_status ht_sync(dhs_table* t);

/* *n_rows = number of keys (= rows) in the table.  Synchronises like ht_sync
 * and returns its status. */
dhs_status ht_size(dhs_table* t, int64_t* n_rows);

/* Synchronous export in row order: h_keys[r] = the key whose offset is r,
 * h_rows[r * stride ..] = its row (weights then state).  Buffers hold at
 * least ht_size rows; either pointer may be NULL. */
dhs_status ht_export(dhs_table* t, int64_t* h_keys, float* h_rows);

/* Counters since creation (synchronises): out[0] rows, out[1] keys inserted
 * by forward / lookup-or-insert calls, out[2] sum over backward calls of the
 * distinct keys updated, out[3] forward-type calls, out[4] backward calls,
 * out[5] IDMap slots, out[6] blocks allocated, out[7] IDMap rehashes,
 * out[8] kernels launched by the table's calls, out[9] keys inserted by the
 * last insert call, out[10] / out[11] times / ns the host waited for the
 * device inside table calls, out[12] / out[13] device allocations / ns spent
 * in them. */
dhs_status ht_counters(dhs_table* t, int64_t out[14]);

/* Per-phase device time, measured with CUDA events recorded on the call's
 * stream around each phase while enabled.  Phases: 0 forward pool (with the
 * probe when bags are short), 1 forward offset assignment + row init,
 * 2 backward probe, 3 backward sort, 4 backward segment reduce + update,
 * 5 lookup-or-insert, 6 IDMap growth, 7 forward probe (long bags: the probe
 * runs as its own kernel before the assignment), 8 backward combine of rows
 * that span three or more sort chunks.
 * enable: 0 off, 1 every phase, 2 the IDMap growth phase only (rare; its
 * events stay out of the launches of the steady-state phases, between which
 * an event delays the next kernel's launch).  Other values: invalid.
 * ht_phase_times synchronises, writes ms_out[p] = total ms and
 * count_out[p] = number of timed launches of phase p (p < n), then clears. */
dhs_status ht_set_phase_timing(dhs_table* t, int enable);
dhs_status ht_phase_times(dhs_table* t, double* ms_out, int64_t* count_out, int n);

/* ---- hash-sharded engine ([RecIS] code-architecture section: collective
 * All-to-All for parameter aggregation; [DLRM-E] practice cases 1 and 2: rows
 * split across cards, lookups exchanged by all-to-all) ----
 * Each of `world` ranks holds one table; key k belongs to rank
 *   owner(k) = floor(hi32(mix(k XOR 0x5DEECE66D)) * world / 2^32),
 * mix = the splitmix64 finaliser (Steele, Lea & Flood; Vigna), hi32 = its
 * upper 32 bits, so that the owner is independent of the IDMap's bucket
 * hash.  One step on a rank:
 *   forward:  ht_shard_route -> exchange the keys (all-to-all) -> each owner
 *             embbag_forward_ex(received keys, one id per bag) gives their
 *             rows -> exchange the rows back -> ht_shard_pool;
 *   backward: ht_shard_grads -> exchange gradient rows and factors -> each
 *             owner embbag_backward_update_ex(received keys, one id per bag,
 *             factors, DHS_POOL_SUM or DHS_POOL_DIVIDE).
 * The exchange is the caller's (NCCL all-to-all in the Python engine).
 * Owners receive the ids in (source rank, position) order, so every sum runs
 * over the terms of the global batch (rank 0's ids first) in that order:
 * pooled outputs are formed as one table forms them (bit for bit from the
 * same rows), and each key's gradient is the fp64 sum one table fed the
 * concatenated batches forms, up to the association of its partial sums. */

/* Route the ids of one batch: d_send_keys int64[n_keys] (device) gets the
 * keys grouped by owner (rank 0's first), in position order within a
 * group; d_slot_of int32[n_keys] (device) gets each position's index in
 * d_send_keys; h_send_counts int64[world] (host) the group sizes.  world in
 * [1, 256]; n_keys < 2^31.  Synchronises the stream (the counts are read on
 * the host).  Uses the table's backward workspace (stream-ordered). */
dhs_status ht_shard_route(dhs_table* t, const int64_t* d_keys, int64_t n_keys, int32_t world,
                          int64_t* d_send_keys, int32_t* d_slot_of, int64_t* h_send_counts, dhs_stream stream);

/* Pool the rows returned by the owners: d_rows float[n_keys, dim] in
 * d_send_keys order; pooled[b] is formed from d_rows[d_slot_of[i]] for the
 * positions i of bag b exactly as embbag_forward_ex forms it from the
 * table's rows (same order, same rounding; mode DHS_POOL_SUM with optional
 * d_per_sample_weights, or DHS_POOL_MEAN).  d_pooled_out float[n_bags, dim]. */
dhs_status ht_shard_pool(dhs_table* t, const float* d_rows, const int32_t* d_slot_of, int64_t n_keys,
                         const int64_t* d_bag_offsets, int64_t n_bags, const float* d_per_sample_weights,
                         dhs_pool_mode mode, float* d_pooled_out, dhs_stream stream);

/* The per-id gradient rows to send to the owners: d_send_grads[d_slot_of[i]]
 * = d_grad[bag(i)] (float[n_keys, dim], copied exactly) and, unless d_send_fact
 * is NULL, d_send_fact[d_slot_of[i]] = the id's factor: its per-sample weight
 * (DHS_POOL_SUM with weights) or its bag's length (DHS_POOL_MEAN, which the
 * owner passes on as DHS_POOL_DIVIDE).  Plain sum pooling needs no factors. */
dhs_status ht_shard_grads(dhs_table* t, const float* d_grad, const int64_t* d_bag_offsets, int64_t n_bags,
                          int64_t n_keys, const int32_t* d_slot_of, const float* d_per_sample_weights,
                          dhs_pool_mode mode, float* d_send_grads, float* d_send_fact, dhs_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* DHS_H_ */

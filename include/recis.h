/*
 * recis.h -- C ABI of the B200 dynamic-hash embedding engine.
 *
 * The library implements the hot path of the RecIS Embedding Engine as the
 * RecIS README describes it (page "RecIS (Recommendation Intelligence
 * System)", codehub.bot mirror of github.com/alibaba/RecIS v1.1.0):
 *   - Core architecture > Feature Engine: Hash / Mod / Bucketize feature ops,
 *     fused into one operator;
 *   - Key optimisations > Efficient dynamic embedding: a two-level store, the
 *     IDMap (feature ID -> offset) and the EmbeddingBlocks (contiguous chunked
 *     memory holding the embedding parameters and the optimiser state,
 *     growing on demand);
 *   - Key optimisations > Distributed optimisation: same-attribute tables merged
 *     into one logical table; requests merged and deduplicated before lookup;
 *   - Key optimisations > Efficient use of hardware > Operator implementation:
 *     vectorised memory access, and reductions merged at warp level instead of
 *     per-element atomics.
 *
 * Conventions (all entry points):
 *   - Every call returns a recis_status and never aborts the process.  Kernels
 *     never trap: device-detected problems set a status word in the table.
 *   - Calls are asynchronous and ordered on the cudaStream_t they are given,
 *     unless marked "synchronous".  Calls on one table (or one batch) must be
 *     issued on one stream, or otherwise serialised by the caller.
 *   - Device pointers are raw CUDA device addresses owned by the caller; they
 *     must stay valid until the work of the call has finished on the stream.
 *     Host pointers are plain host memory, read before the call returns.
 *   - Device arrays are moved with vector loads and copies, so they must be
 *     aligned: float row arrays (pooled and unpooled rows, gradients) to 16
 *     bytes, int64 arrays (keys, offsets, rows) to 8, int32 arrays to 4.  A
 *     misaligned pointer is rejected on the host with RECIS_ERR_INVALID_ARG
 *     before any work is queued.
 *   - Device-detected errors (reserved key, table full, value too wide for its
 *     tag) are reported by recis_table_status_sync(), and by the first later
 *     call on the same table that finds the earlier work finished.
 *   - Keys are int64.  The value -1 (all bits set) is reserved as the IDMap's
 *     empty marker and is rejected (RECIS_ERR_RESERVED_KEY).
 *   - recis_last_error_string() returns a description of the last error of the
 *     calling thread.
 */
#ifndef RECIS_H
#define RECIS_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* recis_stream_t; /* == cudaStream_t; NULL = legacy default stream */

typedef enum {
  RECIS_OK = 0,
  RECIS_ERR_INVALID_ARG = 1,  /* bad argument, or a value wider than its tag field */
  RECIS_ERR_OOM = 2,          /* device or host allocation failed */
  RECIS_ERR_TABLE_FULL = 3,   /* IDMap probe sequence exhausted or row space exhausted */
  RECIS_ERR_RESERVED_KEY = 4, /* an input key equals -1 */
  RECIS_ERR_CUDA = 5,         /* a CUDA runtime/driver call failed */
  RECIS_ERR_TIMEOUT = 6,      /* a bounded device-side wait gave up */
  RECIS_ERR_NO_DEVICE = 7     /* no usable sm_100 device */
} recis_status;

/* ------------------------------------------------------------------ features */
/* Feature-op flags (README, Core architecture > Feature Engine: "Hash / Mod /
 * Bucketize").  Per value x of a feature, in this order:
 *   BUCKETIZE: v = number of boundaries <= x (boundaries sorted ascending);
 *              with FLOAT, x and the boundaries are IEEE-754 binary64 values
 *              stored as their bit patterns in the int64 words and compared
 *              as doubles (-0.0 equals 0.0; a NaN x is above no boundary,
 *              v = 0; the boundaries must hold no NaN);
 *   otherwise: v = (uint64)x; HASH: v = H(v ^ hash_seed); MOD: v = v % mod;
 *   TAG      : v must be < 2^tag_shift, key = (tag << tag_shift) | v.
 * H is the SplitMix64 finaliser (Steele, Lea & Flood, OOPSLA 2014).
 * BUCKETIZE cannot be combined with HASH or MOD; FLOAT needs BUCKETIZE. */
#define RECIS_BUCKETIZE 1u
#define RECIS_HASH 2u
#define RECIS_MOD 4u
#define RECIS_TAG 8u
#define RECIS_FLOAT 16u

typedef struct {
  uint32_t flags;
  int32_t n_bound;            /* number of boundaries (BUCKETIZE) */
  uint64_t hash_seed;
  uint64_t mod;               /* > 0 when MOD is set */
  uint64_t tag;               /* < 2^(63 - tag_shift) */
  int32_t tag_shift;          /* 1..62 */
  int32_t reserved_;
  const int64_t* boundaries;  /* DEVICE pointer, n_bound int64 (binary64 bit patterns with
                                 FLOAT), sorted ascending, 8-byte aligned */
} recis_feature_op;

/* Fused feature transform of F features in one launch.
 * values   : device int64[N], feature-major (feature f occupies
 *            [feat_offsets[f], feat_offsets[f+1]));
 * feat_offsets: HOST int64[F+1], non-decreasing, feat_offsets[0] = 0;
 * keys_out : device int64[N] (may alias values).
 * A transformed value wider than 2^tag_shift is a device-detected error
 * (RECIS_ERR_INVALID_ARG via recis_feature_status_sync); its key is written
 * as -1.  Up to 4096 features per call. */
recis_status recis_feature_hash(const recis_feature_op* ops, int32_t F, const int64_t* values,
                                const int64_t* feat_offsets, int64_t* keys_out,
                                recis_stream_t stream);
/* Synchronous: waits for `stream`, returns and clears the device-detected
 * status of earlier recis_feature_hash calls on the current device. */
recis_status recis_feature_status_sync(recis_stream_t stream);

/* ------------------------------------------------------------------ tables */
#define RECIS_ADAGRAD 0
#define RECIS_ADAM 1
#define RECIS_SUM 0
#define RECIS_MEAN 1

typedef struct {
  int32_t dim;               /* D: multiple of 4, 4..1024 */
  int32_t optimizer;         /* RECIS_ADAGRAD (state: acc) or RECIS_ADAM (state: m, v) */
  double lr;
  double beta1, beta2;       /* Adam */
  double eps;                /* Adagrad 1e-10, Adam 1e-8 are the usual values */
  double adagrad_init_acc;   /* initial accumulator */
  double init_scale;         /* rows start uniform in [-init_scale, init_scale); <= 0: 1/sqrt(D) */
  uint64_t init_seed;
  int64_t initial_capacity;  /* expected live keys; the IDMap starts at >= 2x this */
  int64_t block_rows;        /* rows per EmbeddingBlock (growth unit); 0 = 65536 */
  int64_t max_rows;          /* upper bound on live rows (address space reserved); 0 = 2^28 */
  int32_t admit_threshold;   /* admission: lookups a new key must appear in before it gets a
                                row (0 or 1: at once; at most 65535) */
  int32_t evictable;         /* 1: keep each row's last-lookup clock for recis_table_evict */
  int32_t placement;         /* RECIS_PLACE_* flags: where the table's memory lives (0: all in HBM) */
  int32_t reserved_;
} recis_table_config;

/* Placement (README, Key optimisations > Efficient dynamic embedding: the
 * IDMap and the EmbeddingBlocks can be kept in GPU or in CPU memory).
 *   RECIS_PLACE_BLOCKS_HOST: EmbeddingBlocks (rows, row keys, last-lookup
 *     clocks) are allocated in host memory of the GPU's NUMA node and mapped
 *     into the same contiguous virtual range, so kernels reach them over the
 *     host link with no change; tables beyond HBM fit, at host-link speed.
 *     Needs the driver's host-NUMA support for virtual-memory mappings.
 *   RECIS_PLACE_IDMAP_HOST: the IDMap slot array is mapped pinned host
 *     memory.  Needs native GPU atomics on host memory (the insert is a CAS).
 * A placement the system cannot provide gives RECIS_ERR_INVALID_ARG at
 * create, with the reason in recis_last_error_string(). */
#define RECIS_PLACE_BLOCKS_HOST 1
#define RECIS_PLACE_IDMAP_HOST 2

typedef struct recis_table* recis_table_t;
typedef struct recis_batch* recis_batch_t;

/* Table merging at model-creation time (README, Key optimisations >
 * Distributed optimisation > parameter aggregation: tables with the same
 * attributes -- dimension, initialiser and so on -- are merged into one logical
 * table, so one lookup serves them all).  Host only, synchronous, no GPU.
 * feats[f].table holds feature f's own table attributes; features whose
 * dim, optimizer, lr, beta1, beta2, eps, adagrad_init_acc, init_scale and
 * init_seed are all equal share a logical table.  Tables are numbered in the
 * order their first feature appears; a table's features keep their order.
 * Outputs, per feature f: table_of_feature[f]; tag_of_feature[f] = its rank
 * among its table's features (0, 1, ...); tag_shift_of_feature[f] = the
 * largest value_bits of its table's features -- the RECIS_TAG op's tag and
 * tag_shift that keep the features' IDs apart in the merged table.  Per table
 * t < *n_tables_out: tables_out[t] = the shared attributes, with
 * initial_capacity the sum over its features and max_rows their sum (0 if
 * any feature's is 0).  All output arrays have room for F entries.  Returns
 * RECIS_ERR_INVALID_ARG for value_bits outside 1..62 or when a table has more
 * features than 2^(63 - tag_shift) tags. */
typedef struct {
  recis_table_config table;  /* the feature's own table attributes */
  int32_t value_bits;        /* its transformed values are < 2^value_bits (1..62) */
  int32_t reserved_;
} recis_feature_spec;
recis_status recis_plan_tables(const recis_feature_spec* feats, int32_t F,
                               int32_t* table_of_feature, uint64_t* tag_of_feature,
                               int32_t* tag_shift_of_feature, recis_table_config* tables_out,
                               int32_t* n_tables_out);

/* Admission and eviction (README, Core architecture > Embedding Engine: the
 * table supports feature eviction and admission policies; the README names no
 * policy, so these are the readings):
 *   - Admission: a key not in the table is a candidate.  Each lookup it appears
 *     in (however often) raises its count by one; the lookup that brings the
 *     count to admit_threshold gives it a row (new rows in ascending key order,
 *     as always).  Until then its occurrences pool as zero vectors (MEAN still
 *     divides by the whole bag length), its unpooled rows are zeros, its
 *     gradient is dropped, and recis_batch_get_unique reports row -1 for it.
 *     Candidates live in IDMap slots only; they use no EmbeddingBlock row.
 *   - Clock: every lookup or insert that launches work advances the table's
 *     clock by one; an evictable table records in each row (and each
 *     candidate) the clock of the last lookup that touched it.
 *   - Eviction: recis_table_evict removes every row and candidate last touched
 *     before a given clock.  An evicted key keeps its IDMap slot as a
 *     tombstone (so no probe chain is cut) until an IDMap growth drops it; if
 *     it comes back it starts over as a new candidate with an initial row.
 *     Freed rows (key -1) join a queue in ascending row order; later new keys
 *     take them, oldest first, before rows past the end.  Exports, saves and
 *     recis_table_size count live rows only. */

/* Create a table on the current device (README, Efficient dynamic embedding:
 * IDMap + EmbeddingBlocks).  Rows are [emb D][state s*D] fp32 (s = 1 Adagrad,
 * 2 Adam), kept side by side in EmbeddingBlocks that are physically separate
 * allocations mapped into one contiguous virtual range, so a row is addressed
 * as base + row * stride and growth never copies.  *out receives the handle. */
recis_status recis_table_create(const recis_table_config* cfg, recis_stream_t stream,
                                recis_table_t* out);
recis_status recis_table_destroy(recis_table_t t);

/* A batch holds the per-step scratch of one lookup (sorted keys, unique keys,
 * inverse index, row offsets, per-occurrence bag ids) until the matching
 * backward; it grows on demand and is reused across steps. */
recis_status recis_batch_create(recis_batch_t* out);
recis_status recis_batch_destroy(recis_batch_t b);

/* Forward (README, Distributed optimisation: merged requests deduplicated; Efficient
 * dynamic embedding: IDMap lookup, then the EmbeddingBlocks rows).  One call =
 * one logical table:
 *   1. dedup: uniq = distinct keys ascending (signed), inv[i] = index of keys[i];
 *   2. IDMap find-or-insert: a missing key gets the next free row; new rows are
 *      assigned in ascending key order and initialised from a seeded hash of
 *      the key (emb) and the optimiser's initial state;
 *   3. pooling: bag f*B+b covers keys[bag_offsets[f*B+b] .. bag_offsets[f*B+b+1]);
 *      pooled_out[b][f][:] = sum of its rows (MEAN: / length; empty bag: 0);
 *      unpooled_out[i][:] = row of keys[i].
 * keys: device int64[N]; bag_offsets: device int64[F*B+1] (0 .. N, non-decreasing);
 * pooled_out: device fp32 [B][F][D] or NULL; unpooled_out: device fp32 [N][D]
 * or NULL.  keys and bag_offsets must stay unchanged until the matching
 * recis_backward_update has run.  0 <= N < 2^30 (larger N: RECIS_ERR_INVALID_ARG).
 * A lookup whose keys include the reserved -1 is rejected as a whole: no key
 * is inserted, no row is created, the table is left as it was, and
 * RECIS_ERR_RESERVED_KEY is reported as a device-detected error.  Batches of
 * up to 1,600,000 keys are rejected the same way (RECIS_ERR_TABLE_FULL) when
 * their new keys would not fit in max_rows; for larger batches the host checks
 * the bound live rows + N against max_rows before launching and returns
 * RECIS_ERR_TABLE_FULL at once.  The outputs of a rejected lookup are
 * undefined and its recis_backward_update updates no row. */
recis_status recis_lookup_pooled(recis_table_t t, recis_batch_t b, const int64_t* keys,
                                 int64_t N, const int64_t* bag_offsets, int32_t F, int64_t B,
                                 int32_t combiner, float* pooled_out, float* unpooled_out,
                                 recis_stream_t stream);

/* Backward + optimiser for the batch's last lookup (README, Operator
 * implementation: reduction merged at warp level; Efficient dynamic embedding:
 * optimiser state beside the parameters).  g(u) = sum over occurrences of
 * key u of grad_pooled[b][f] (x 1/length for MEAN) + grad_unpooled[i], then one
 * Adagrad or Adam step on every row touched by the lookup (Adam: the table's
 * step counter advances by one per call).  grad_pooled: [B][F][D] or NULL;
 * grad_unpooled: [N][D] or NULL (NULL = zero gradient); 16-byte aligned,
 * unchanged until the call's work has finished.  They are normally device
 * memory (gathered by the bulk-copy engine); any memory the GPU can read
 * (host-mapped pinned memory, managed memory) is accepted and gathered with
 * per-thread copies instead.  A gradient of several occurrences is summed in
 * fp64 in a fixed order and rounded once, so results do not depend on
 * scheduling. */
recis_status recis_backward_update(recis_table_t t, recis_batch_t b, const float* grad_pooled,
                                   const float* grad_unpooled, recis_stream_t stream);

/* Find-or-insert only (no pooling): used to pre-load a table; its keys are
 * admitted at once whatever the admission threshold.  keys: device int64[N].
 * rows_out: device int64[N] (row of each key) or NULL. */
recis_status recis_table_insert(recis_table_t t, recis_batch_t b, const int64_t* keys, int64_t N,
                                int64_t* rows_out, recis_stream_t stream);

/* Row access by offset (README, Efficient dynamic embedding: parameters and
 * optimiser state kept side by side).  For each of the n row offsets rows[i]
 * (device int64[n]) writes its key to keys_out[i] (device int64[n] or NULL),
 * its emb to emb_out[i][0..D) (device fp32 [n][D] or NULL) and its optimiser
 * state to state_out[i][0..s*D) (device fp32 [n][s*D] or NULL; Adam: m then
 * v).  A row offset outside [0, rows in use) gives key -1 and zeros; a row
 * freed by eviction and not yet reused gives key -1 (its values are left
 * over from its last key).  Waits for
 * `stream` to learn the live row count, then gathers asynchronously on it. */
recis_status recis_table_read_rows(recis_table_t t, const int64_t* rows, int64_t n,
                                   int64_t* keys_out, float* emb_out, float* state_out,
                                   recis_stream_t stream);

/* Synchronous.  Makes room for `rows` live rows in total (README, Efficient
 * dynamic embedding: EmbeddingBlocks grow on demand): maps EmbeddingBlocks and
 * sizes the IDMap for them now, so that lookups that keep the table at or
 * below that many rows map nothing and rehash nothing while they run (a
 * lookup may still wait for earlier work when its host-side bound on new rows
 * says it could pass the mapped rows).  Waits for `stream` first and returns
 * any pending device-detected error.  rows > max_rows: RECIS_ERR_TABLE_FULL. */
recis_status recis_table_reserve(recis_table_t t, int64_t rows, recis_stream_t stream);

/* Synchronous (README, Core architecture > Embedding Engine: feature eviction).
 * Evicts every row and candidate whose last lookup clock is below min_clock
 * (rows touched by the lookups numbered min_clock and later stay); *n_evicted
 * (may be NULL) receives the number of rows freed.  The table must have been
 * created with evictable = 1 (else RECIS_ERR_INVALID_ARG).  *clock_out of
 * recis_table_clock is the number of lookups so far. */
recis_status recis_table_evict(recis_table_t t, int64_t min_clock, int64_t* n_evicted,
                               recis_stream_t stream);
recis_status recis_table_clock(recis_table_t t, int64_t* clock_out);

/* Synchronous.  Number of live rows and the Adam step counter. */
recis_status recis_table_size(recis_table_t t, int64_t* n_out, int64_t* step_out,
                              recis_stream_t stream);

/* Synchronous (README, Core architecture > Saver: sparse parameters saved for
 * delivery).  Copies the first min(n, capacity) rows, in ascending row order,
 * to HOST buffers: keys int64[capacity] (or NULL), emb fp32 [capacity][D] (or
 * NULL), state fp32 [capacity][s*D] (or NULL; Adam: m then v).  *n_out = live
 * rows, *step_out = Adam step. */
recis_status recis_table_export(recis_table_t t, int64_t* keys, float* emb, float* state,
                                int64_t capacity, int64_t* n_out, int64_t* step_out,
                                recis_stream_t stream);

/* Synchronous (README, Core architecture > Saver: sparse parameters stored and
 * delivered in the SafeTensors standard format).  Writes the table to the file
 * `path` in the SafeTensors format: tensors "keys" (I64 [n]), "emb" (F32 [n, D])
 * and the optimiser state, "accum" (Adagrad) or "adam_m" and "adam_v" (Adam),
 * each F32 [n, D], rows in ascending row order; metadata "format" =
 * "recis-embedding-table", "dim", "optimizer", "step", "rows", "lr", "beta1",
 * "beta2", "eps", "adagrad_init_acc", "init_scale", "init_seed" (strings).  The
 * rows stream through host memory in chunks of about 64 MB.  An unwritable path
 * gives RECIS_ERR_INVALID_ARG. */
recis_status recis_table_save(recis_table_t t, const char* path, recis_stream_t stream);
/* Synchronous.  Reads a SafeTensors file holding "keys", "emb" and this table's
 * optimiser-state tensors (as recis_table_save writes them) with dim D and
 * appends its rows after the live rows, as recis_table_import does (keys must
 * be new); the metadata "step", when present, becomes the table's step
 * counter.  A file without those tensors, or with another dim, gives
 * RECIS_ERR_INVALID_ARG and leaves the table unchanged. */
recis_status recis_table_load(recis_table_t t, const char* path, recis_stream_t stream);

/* Synchronous.  Appends n rows from HOST buffers after the live rows (keys must
 * not be present; state NULL = initial state) and sets the step counter. */
recis_status recis_table_import(recis_table_t t, const int64_t* keys, const float* emb,
                                const float* state, int64_t n, int64_t step,
                                recis_stream_t stream);

/* Synchronous: waits for `stream`; returns and clears the table's device status. */
recis_status recis_table_status_sync(recis_table_t t, recis_stream_t stream);

/* Synchronous.  Copies the last lookup's dedup into caller DEVICE buffers (each
 * may be NULL): uniq_out int64[capacity] (the min(U, capacity) unique keys,
 * ascending), rows_out int64[capacity] (their row offsets), inv_out int32[N]
 * (index into uniq of every key).  *U_out = U, *n_new_out = keys inserted. */
recis_status recis_batch_get_unique(recis_batch_t b, int64_t* uniq_out, int32_t* inv_out,
                                    int64_t* rows_out, int64_t capacity, int64_t* U_out,
                                    int64_t* n_new_out, recis_stream_t stream);

/* Dedup without any allocation.  The pages have no counterpart: this exists for
 * callers that cannot allocate device memory (code inside a framework whose
 * memory pool forbids foreign cudaMalloc calls, work recorded into a graph
 * with allocation disabled, or a process that budgets its device memory up
 * front), which cannot use recis_lookup_pooled because a recis_batch_t grows
 * its scratch with cudaMalloc.  Computes the same dedup as the first step of
 * recis_lookup_pooled: uniq_out = distinct keys ascending (signed), inv_out[i]
 * = index of keys[i] in uniq_out, *U_out = number of unique keys (-1 if a
 * bounded device-side wait gave up).  Any int64 key is allowed, -1 included
 * (no IDMap is involved).
 *   keys: device int64[N], 0 <= N <= 262144 (larger N: RECIS_ERR_INVALID_ARG);
 *   uniq_out: device int64[N]; inv_out: device int32[N]; U_out: device int64[1].
 * Asynchronous on `stream`; no cudaMalloc, cudaFree or allocating library call.
 * Its scratch is one fixed __device__ array of about 6.3 MB that every GPU
 * which loads the library holds until the process exits.  The first call on a
 * device looks up that array's device address (cudaGetSymbolAddress); make
 * that first call before any stream capture.  All calls share the array and
 * clear what must start at zero themselves; calls that overlap on the GPU
 * (different streams, or several host threads) race and must be serialised by
 * the caller. */
recis_status recis_unique_static(const int64_t* keys, int64_t N, int64_t* uniq_out,
                                 int32_t* inv_out, int64_t* U_out, recis_stream_t stream);

/* ------------------------------------------------------------------ sharded tables */
/* Building blocks of tables sharded over GPUs (README, Key optimisations >
 * Distributed optimisation: parameters split evenly over the nodes; each node
 * merges and deduplicates its requests and fetches the embeddings from their
 * owners with an All-to-All).  A requesting GPU dedups its batch, groups the
 * unique keys by owner, exchanges them (an NCCL all-to-all issued by the
 * caller), pools the rows that come back, and in the backward sends each
 * unique key's summed gradient to its owner, which applies it with
 * recis_backward_update as an unpooled gradient of a lookup that had one bag
 * per received key.  All asynchronous on `stream` unless marked synchronous.
 *
 * recis_batch_dedup: uniq_out (device int64[N]) = distinct keys ascending,
 *   inv_out (device int32[N]) = index of keys[i] in uniq_out, *U_out (device
 *   int64) = their number (-1 if a bounded wait gave up).  The batch keeps
 *   the grouping of occurrences by unique key for recis_reduce_grad; any int64
 *   key is allowed.  0 <= N < 2^30.
 * recis_partition_keys (synchronous): a stable partition of keys[0..n) by
 *   owner = H(key ^ salt) mod G (H: the SplitMix64 finaliser): out_keys
 *   (device int64[n]) holds the keys of owner 0, then owner 1, ..., each in
 *   input order; out_pos[i] (device int32[n]) = where keys[i] went;
 *   counts_out (device int64[G]) = keys per owner.  1 <= G <= 256.
 * recis_pool_rows: pooled_out[b][f] = sum (MEAN: / bag length; empty bag: 0)
 *   over the occurrences i of bag f*B+b of rows[r(inv[i])], r(u) =
 *   row_of_unique[u] (device int32, or NULL for u); rows: device fp32
 *   [*][D]; fp64 sums rounded once.
 * recis_reduce_grad: for every unique key u of the batch's last
 *   recis_batch_dedup, g(u) = the sum over its occurrences i of
 *   grad_pooled[bag(i)] (x 1/length for MEAN) + grad_unpooled[i] (either may
 *   be NULL), in occurrence order in fp64, rounded once, written to
 *   grad_out[o(u)][0..D), o(u) = out_index[u] (device int32, or NULL for u). */
recis_status recis_batch_dedup(recis_batch_t b, const int64_t* keys, int64_t N, int64_t* uniq_out,
                               int32_t* inv_out, int64_t* U_out, recis_stream_t stream);
recis_status recis_partition_keys(recis_batch_t b, const int64_t* keys, int64_t n, int32_t G,
                                  uint64_t salt, int64_t* out_keys, int32_t* out_pos,
                                  int64_t* counts_out, recis_stream_t stream);
recis_status recis_pool_rows(const float* rows, const int32_t* row_of_unique, const int32_t* inv,
                             const int64_t* bag_offsets, int32_t F, int64_t B, int32_t D,
                             int32_t combiner, float* pooled_out, recis_stream_t stream);
recis_status recis_reduce_grad(recis_batch_t b, const int64_t* bag_offsets, int32_t F, int64_t B,
                               int32_t D, int32_t combiner, const float* grad_pooled,
                               const float* grad_unpooled, const int32_t* out_index,
                               float* grad_out, recis_stream_t stream);

/* ------------------------------------------------------------------ test hooks */
/* Process-wide settings that let tests reach error paths without faulting the
 * GPU.  The pages have no counterpart (they describe no failure handling).
 *   RECIS_DEBUG_SPIN_LIMIT: polls a device-side wait on another CTA's progress
 *     makes before it gives up and reports RECIS_ERR_TIMEOUT (value 0 restores
 *     the default, about 4M polls).  Applies to launches made after the call:
 *     the radix-sort dedup of batches over 1.6M keys and recis_unique_static.
 *     A wait that gives up leaves the call's outputs undefined (every access
 *     stays in bounds); on a table it also leaves the table's contents
 *     undefined.
 *   RECIS_DEBUG_MAP_LIMIT: EmbeddingBlock bytes one table may have mapped;
 *     growth past it fails with RECIS_ERR_OOM as a failed allocation would
 *     (0 = no cap, the default).
 * Returns RECIS_ERR_INVALID_ARG for an unknown setting or a negative value. */
#define RECIS_DEBUG_SPIN_LIMIT 1
#define RECIS_DEBUG_MAP_LIMIT 2
recis_status recis_debug_set(int32_t what, int64_t value);

/* ------------------------------------------------------------------ tracing */
/* Kernel timing: while enabled, every kernel launch is bracketed by CUDA
 * events on its stream.  recis_profile_collect (synchronous) returns per kernel
 * name: launches and total milliseconds, clears the record, and returns the
 * number of names (<= max).  recis_launch_count counts all kernel launches of
 * the library since load. */
recis_status recis_profile_enable(int32_t on);
int32_t recis_profile_collect(const char** names, int64_t* launches, double* total_ms,
                              int32_t max);
int64_t recis_launch_count(void);

const char* recis_last_error_string(void);

#ifdef __cplusplus
}
#endif
#endif

/*
 * oracle.h -- plain, slow, single-threaded CPU oracle of the RecIS dynamic-hash
 * embedding step.  TEST INFRASTRUCTURE ONLY: only the tests, the smoke check and
 * the benchmark's CPU-baseline leg may load it.  It shares no code, header,
 * constant or helper with the CUDA library.
 *
 * What it follows (RecIS README, "Core architecture" and "Key optimisations"):
 *   - Feature Engine: Hash / Mod / Bucketize feature transforms.
 *   - Embedding Engine, "Efficient dynamic embedding": a first-level IDMap
 *     (feature ID -> offset) and second-level EmbeddingBlocks that hold the
 *     embedding parameters and the optimiser state side by side.
 *   - "Distributed optimisation": same-attribute tables merged into one logical
 *     table; requests merged and deduplicated before the lookup.
 *   - "Operator optimisation": a reduction of the gradients per unique ID.
 * Readings where the pages are silent (hash function, tag layout, row order,
 * initialiser, optimiser formulas) are listed at each function in oracle.cpp.
 *
 * Arithmetic: integer work is exact; floating point accumulates in double and
 * rounds once to fp32 when it is stored (the table itself is fp32).
 */
#ifndef RECIS_ORACLE_H
#define RECIS_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* status codes of the oracle (its own numbering) */
#define ORC_OK 0
#define ORC_INVALID_ARG 1
#define ORC_RESERVED_KEY 2

/* feature-op flags */
#define ORC_BUCKETIZE 1u
#define ORC_HASH 2u
#define ORC_MOD 4u
#define ORC_TAG 8u
#define ORC_FLOAT 16u /* with ORC_BUCKETIZE: values and boundaries are IEEE binary64 bit patterns */

typedef struct {
  uint32_t flags;
  int32_t n_bound;            /* number of bucket boundaries */
  uint64_t hash_seed;         /* xor-ed into the value before hashing */
  uint64_t mod;               /* modulus (> 0) for ORC_MOD */
  uint64_t tag;               /* feature tag written above tag_shift */
  int32_t tag_shift;          /* bit position of the tag, 1..62 */
  int32_t pad_;
  const int64_t* boundaries;  /* host, sorted ascending, n_bound entries (binary64 bits with ORC_FLOAT) */
} orc_feature_op;

#define ORC_ADAGRAD 0
#define ORC_ADAM 1
#define ORC_SUM 0
#define ORC_MEAN 1

typedef struct orc_table orc_table;

uint64_t orc_hash64(uint64_t x);

int orc_feature_hash(const orc_feature_op* ops, int32_t F, const int64_t* values,
                     const int64_t* feat_offsets, int64_t* keys_out);

orc_table* orc_table_new(int32_t dim, int32_t optimizer, double lr, double beta1,
                         double beta2, double eps, double adagrad_init_acc,
                         uint64_t init_seed, double init_scale);
void orc_table_free(orc_table* t);

/* Forward of one batch.  keys[N]; bags are feature-major (bag f*B+b covers
 * keys[bag_offsets[f*B+b] .. bag_offsets[f*B+b+1])).  pooled_out is [B][F][D]
 * or NULL, unpooled_out is [N][D] or NULL.  uniq_out/rows_out have room for N,
 * inv_out is [N].  The batch is remembered for orc_backward_update. */
int orc_lookup(orc_table* t, const int64_t* keys, int64_t N, const int64_t* bag_offsets,
               int32_t F, int64_t B, int32_t combiner, float* pooled_out,
               float* unpooled_out, int64_t* uniq_out, int32_t* inv_out,
               int64_t* rows_out, int64_t* U_out, int64_t* n_new_out);

/* Backward + optimiser for the last batch.  grad_pooled [B][F][D] or NULL,
 * grad_unpooled [N][D] or NULL (NULL = zero gradient). grad_u_out [U][D] or
 * NULL receives the reduced gradient per unique key (double, before rounding). */
int orc_backward_update(orc_table* t, const float* grad_pooled, const float* grad_unpooled,
                        double* grad_u_out);

/* live rows (rows freed by eviction excluded) */
int64_t orc_table_size(const orc_table* t);
int64_t orc_table_step(const orc_table* t);
/* lookups so far (the clock eviction compares against) */
int64_t orc_table_clock(const orc_table* t);
/* admission: a key gets a row on the lookup that brings its count of lookups
 * seen in to `threshold` (0 or 1: at once) */
int orc_table_set_admission(orc_table* t, int32_t threshold);
/* eviction: rows and candidates last touched by a lookup before min_clock are
 * removed; freed rows are reused by later keys, oldest first */
int orc_table_evict(orc_table* t, int64_t min_clock, int64_t* n_evicted);
/* live rows in ascending row order; state is [n][s*D] (s = 1 Adagrad, 2 Adam: m then v) */
int orc_table_export(const orc_table* t, int64_t* keys, float* emb, float* state);
/* append rows (key, emb, state) after the live rows; keys must be new */
int orc_table_import(orc_table* t, int64_t n, const int64_t* keys, const float* emb,
                     const float* state, int64_t step);

/* Table merging (README, Key optimisations > Distributed optimisation >
 * parameter aggregation: tables with the same attributes are merged into one
 * logical table at model-creation time).  Per feature: its table attributes
 * and the bit width of its transformed values.  Outputs per feature: the
 * logical table (numbered by first appearance), the tag (rank among the
 * table's features) and the tag shift (widest value of the table); per table:
 * the summed initial capacity.  Returns ORC_INVALID_ARG when bits are outside
 * 1..62 or a table's tags do not fit above its values. */
typedef struct {
  int32_t dim;
  int32_t optimizer;
  double lr, beta1, beta2, eps, adagrad_init_acc, init_scale;
  uint64_t init_seed;
  int64_t capacity;
  int32_t value_bits;
  int32_t pad_;
} orc_feature_attrs;

int orc_plan_tables(const orc_feature_attrs* feats, int32_t F, int32_t* table_of,
                    uint64_t* tag_of, int32_t* shift_of, int64_t* table_capacity,
                    int32_t* n_tables);

#ifdef __cplusplus
}
#endif
#endif

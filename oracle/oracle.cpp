// oracle.cpp -- the CPU oracle of the RecIS dynamic-hash embedding step.
//
// TEST INFRASTRUCTURE ONLY.  This file is the definition the CUDA library is
// checked against; it is never on the product path and shares no code with it.
// Build: g++ -std=c++17 -O2 -ffp-contract=off -fno-fast-math -shared -fPIC.
//
// Every step is the plain definition, written in the order the method states
// it.  Where the RecIS README is silent the reading taken is stated beside the
// code.  Floating point: sums and optimiser arithmetic in double, one rounding
// to fp32 on store.
#include "oracle.h"

#include <algorithm>
#include <cmath>
#include <cstring>
#include <map>
#include <tuple>
#include <unordered_map>
#include <vector>

namespace {

// H: the SplitMix64 finaliser ("mix64" of Steele, Lea & Flood, "Fast splittable
// pseudorandom number generators", OOPSLA 2014; Stafford's variant 13
// constants).  The README names a "Hash" feature op and no function; this is
// the reading: bijective on 64 bits, integer-only.
uint64_t H(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  return z ^ (z >> 31);
}

const int64_t kReserved = -1;  // the IDMap's empty marker; not a legal key

}  // namespace

struct orc_table {
  int32_t D;
  int32_t opt;  // ORC_ADAGRAD / ORC_ADAM
  int32_t s;    // optimiser state vectors per row
  double lr, beta1, beta2, eps, acc0;
  uint64_t init_seed;
  float init_scale;  // rounded to fp32 once

  // First level: IDMap, feature ID -> row offset (README, Key optimisations,
  // "Efficient dynamic embedding", IDMap bullet).
  std::unordered_map<int64_t, int64_t> idmap;
  // Admission and eviction (README, Core architecture > Embedding Engine: the
  // table supports feature eviction and admission policies).  Reading: a key
  // not in the IDMap is a candidate whose count rises by one per lookup it
  // appears in; it gets a row on the lookup where the count reaches
  // admit_threshold (<= 1: at once).  Every lookup advances the clock; a row
  // (or a candidate) remembers the clock of the last lookup that touched it,
  // and eviction removes those last touched before a given clock.  Freed rows
  // queue in ascending row order and are handed to new keys first.
  int32_t admit_threshold = 1;
  int64_t clock = 0;
  std::unordered_map<int64_t, std::pair<int64_t, int64_t>> cand;  // key -> (count, last clock)
  std::vector<int64_t> last_seen;                                  // per row
  std::vector<int64_t> free_rows;                                  // queue of freed rows
  size_t free_head = 0;
  // Second level: rows of [emb D][state s*D] fp32 in row order
  // (same section, EmbeddingBlocks bullet: parameters and optimiser state kept
  // together).  One flat vector stands for the chunked blocks.
  std::vector<int64_t> row_key;
  std::vector<float> emb;    // [rows][D]
  std::vector<float> state;  // [rows][s*D]
  int64_t step = 0;          // Adam step counter, one per table

  // the last forward batch, kept for the backward pass
  std::vector<int64_t> uniq, rows;
  std::vector<int32_t> inv;
  std::vector<int64_t> bag_offsets;
  int64_t N = 0, B = 0;
  int32_t F = 0;
  int32_t combiner = ORC_SUM;
  bool have_batch = false;
};

extern "C" uint64_t orc_hash64(uint64_t x) { return H(x); }

// Feature transform (README, Core architecture, Feature Engine: Hash / Mod /
// Bucketize).  Per value x of feature f:
//   BUCKETIZE: v = number of boundaries <= x  (reading: upper-bound index);
//              FLOAT: x and the boundaries are binary64 values stored as
//              their bit patterns, compared as doubles (a NaN x is above no
//              boundary: v = 0)
//   else     : v = (uint64)x; HASH: v = H(v ^ seed); MOD: v = v % mod
//   TAG      : v must be < 2^shift; key = (tag << shift) | v
// Reading for TAG: merged tables (Distributed optimisation, "parameter
// aggregation") must keep features apart; the tag in the high bits does that.
extern "C" int orc_feature_hash(const orc_feature_op* ops, int32_t F, const int64_t* values,
                                const int64_t* feat_offsets, int64_t* keys_out) {
  if (F < 0) return ORC_INVALID_ARG;
  for (int32_t f = 0; f < F; ++f) {
    const orc_feature_op& op = ops[f];
    if ((op.flags & ORC_BUCKETIZE) && (op.flags & (ORC_HASH | ORC_MOD))) return ORC_INVALID_ARG;
    if ((op.flags & ORC_MOD) && op.mod == 0) return ORC_INVALID_ARG;
    if ((op.flags & ORC_BUCKETIZE) && op.n_bound < 0) return ORC_INVALID_ARG;
    if ((op.flags & ORC_FLOAT) && !(op.flags & ORC_BUCKETIZE)) return ORC_INVALID_ARG;
    if (op.flags & ORC_TAG) {
      if (op.tag_shift < 1 || op.tag_shift > 62) return ORC_INVALID_ARG;
      if (op.tag >= (1ULL << (63 - op.tag_shift))) return ORC_INVALID_ARG;
    }
    if (feat_offsets[f + 1] < feat_offsets[f]) return ORC_INVALID_ARG;
    for (int64_t i = feat_offsets[f]; i < feat_offsets[f + 1]; ++i) {
      const int64_t x = values[i];
      uint64_t v;
      if ((op.flags & ORC_BUCKETIZE) && (op.flags & ORC_FLOAT)) {
        double xd;
        std::memcpy(&xd, &x, sizeof xd);
        int64_t c = 0;
        for (int32_t k = 0; k < op.n_bound; ++k) {
          double bd;
          std::memcpy(&bd, &op.boundaries[k], sizeof bd);
          if (bd <= xd) ++c;
        }
        v = (uint64_t)c;
      } else if (op.flags & ORC_BUCKETIZE) {
        int64_t c = 0;
        for (int32_t k = 0; k < op.n_bound; ++k)
          if (op.boundaries[k] <= x) ++c;
        v = (uint64_t)c;
      } else {
        v = (uint64_t)x;
        if (op.flags & ORC_HASH) v = H(v ^ op.hash_seed);
        if (op.flags & ORC_MOD) v = v % op.mod;
      }
      if (op.flags & ORC_TAG) {
        if (v >= (1ULL << op.tag_shift)) return ORC_INVALID_ARG;
        v = (op.tag << op.tag_shift) | v;
      }
      keys_out[i] = (int64_t)v;
    }
  }
  return ORC_OK;
}

extern "C" orc_table* orc_table_new(int32_t dim, int32_t optimizer, double lr, double beta1,
                                    double beta2, double eps, double adagrad_init_acc,
                                    uint64_t init_seed, double init_scale) {
  if (dim <= 0 || (optimizer != ORC_ADAGRAD && optimizer != ORC_ADAM)) return nullptr;
  orc_table* t = new orc_table();
  t->D = dim;
  t->opt = optimizer;
  t->s = optimizer == ORC_ADAGRAD ? 1 : 2;
  t->lr = lr;
  t->beta1 = beta1;
  t->beta2 = beta2;
  t->eps = eps;
  t->acc0 = adagrad_init_acc;
  t->init_seed = init_seed;
  t->init_scale = (float)init_scale;
  return t;
}

extern "C" void orc_table_free(orc_table* t) { delete t; }

// Row initialiser.  The README makes the initializer a table attribute
// (Distributed optimisation, tables merged by "dimension, initializer, etc.")
// and names none; reading: a seeded hash of the ID, so that a row depends on
// its key alone and not on when or where it was inserted.
//   h = H(H(key ^ seed) + j);  u = (h >> 40) * 2^-24 in [0, 1)
//   emb[j] = (u - 1/2) * (2 * scale)      (exact in double, rounded once)
//   Adagrad accumulator = init value; Adam m = v = 0.
static void init_row(orc_table* t, int64_t key, int64_t row) {
  const int D = t->D;
  const uint64_t base = H((uint64_t)key ^ t->init_seed);
  const double two_s = 2.0 * (double)t->init_scale;
  for (int j = 0; j < D; ++j) {
    const uint64_t h = H(base + (uint64_t)j);
    const double u = (double)(h >> 40) * (1.0 / 16777216.0);
    t->emb[row * D + j] = (float)((u - 0.5) * two_s);
  }
  for (int j = 0; j < t->s * D; ++j) {
    float v = 0.0f;
    if (t->opt == ORC_ADAGRAD) v = (float)t->acc0;
    t->state[row * t->s * D + j] = v;
  }
}

// A new row at the end of the table.
static int64_t add_row(orc_table* t, int64_t key) {
  const int64_t row = (int64_t)t->row_key.size();
  t->row_key.push_back(key);
  t->emb.resize((size_t)(row + 1) * t->D);
  t->state.resize((size_t)(row + 1) * t->s * t->D);
  t->last_seen.push_back(t->clock);
  t->idmap.emplace(key, row);
  return row;
}

// The row of a key admitted by a lookup: the oldest freed row if any, else a
// new one at the end.
static int64_t take_row(orc_table* t, int64_t key) {
  if (t->free_head < t->free_rows.size()) {
    const int64_t row = t->free_rows[t->free_head++];
    t->row_key[row] = key;
    t->last_seen[row] = t->clock;
    t->idmap.emplace(key, row);
    return row;
  }
  return add_row(t, key);
}

// Forward.  Steps, in order:
//  1. dedup (Distributed optimisation: requests of merged tables are merged and
//     deduplicated).  uniq = the distinct keys in ascending signed order; inv[i]
//     = position of keys[i] in uniq.  (Reading: ascending order makes the unique
//     list and the row assignment canonical.)
//  2. IDMap find-or-insert for each uniq[j] in ascending order; a missing key
//     gets the next free row (rows of new keys therefore follow ascending key
//     order, after all rows of earlier batches) and is initialised.
//  3. pooling per bag: sum of the rows of its keys, or that sum / L for mean;
//     an empty bag gives zeros.  Unpooled: the row of each occurrence.
extern "C" int orc_lookup(orc_table* t, const int64_t* keys, int64_t N, const int64_t* bag_offsets,
                          int32_t F, int64_t B, int32_t combiner, float* pooled_out,
                          float* unpooled_out, int64_t* uniq_out, int32_t* inv_out,
                          int64_t* rows_out, int64_t* U_out, int64_t* n_new_out) {
  if (!t || N < 0 || F < 0 || B < 0) return ORC_INVALID_ARG;
  if (combiner != ORC_SUM && combiner != ORC_MEAN) return ORC_INVALID_ARG;
  const int64_t nbags = (int64_t)F * B;
  if (nbags > 0) {
    if (bag_offsets[0] != 0 || bag_offsets[nbags] != N) return ORC_INVALID_ARG;
    for (int64_t j = 0; j < nbags; ++j)
      if (bag_offsets[j + 1] < bag_offsets[j]) return ORC_INVALID_ARG;
  } else if (N != 0) {
    return ORC_INVALID_ARG;
  }
  t->clock += 1;  // every accepted call advances the clock, even one rejected below
  for (int64_t i = 0; i < N; ++i)
    if (keys[i] == kReserved) return ORC_RESERVED_KEY;

  // 1. dedup
  std::vector<int64_t> uniq(keys, keys + N);
  std::sort(uniq.begin(), uniq.end());
  uniq.erase(std::unique(uniq.begin(), uniq.end()), uniq.end());
  std::vector<int32_t> inv((size_t)N);
  for (int64_t i = 0; i < N; ++i)
    inv[i] = (int32_t)(std::lower_bound(uniq.begin(), uniq.end(), keys[i]) - uniq.begin());

  // 2. find-or-insert
  const int64_t U = (int64_t)uniq.size();
  std::vector<int64_t> rows((size_t)U);
  int64_t n_new = 0;
  for (int64_t j = 0; j < U; ++j) {
    auto it = t->idmap.find(uniq[j]);
    if (it != t->idmap.end()) {
      rows[j] = it->second;
      t->last_seen[rows[j]] = t->clock;
      continue;
    }
    // a candidate: admitted when this lookup brings its count to the threshold
    auto c = t->cand.find(uniq[j]);
    const int64_t count = (c == t->cand.end() ? 0 : c->second.first) + 1;
    if (count >= t->admit_threshold) {
      if (c != t->cand.end()) t->cand.erase(c);
      rows[j] = take_row(t, uniq[j]);
      init_row(t, uniq[j], rows[j]);
      ++n_new;
    } else {
      t->cand[uniq[j]] = std::make_pair(count, t->clock);
      rows[j] = -1;  // no row yet: pooled as zeros, gradient dropped
    }
  }

  // 3. pooling
  const int D = t->D;
  std::vector<double> acc((size_t)D);
  if (pooled_out) {
    for (int32_t f = 0; f < F; ++f) {
      for (int64_t b = 0; b < B; ++b) {
        const int64_t bag = (int64_t)f * B + b;
        std::fill(acc.begin(), acc.end(), 0.0);
        const int64_t lo = bag_offsets[bag], hi = bag_offsets[bag + 1];
        for (int64_t i = lo; i < hi; ++i) {
          if (rows[inv[i]] < 0) continue;  // a candidate's occurrence adds zeros
          const float* e = &t->emb[(size_t)rows[inv[i]] * D];
          for (int j = 0; j < D; ++j) acc[j] += (double)e[j];
        }
        const int64_t L = hi - lo;
        float* o = pooled_out + ((size_t)b * F + f) * D;
        for (int j = 0; j < D; ++j) {
          double v = acc[j];
          if (combiner == ORC_MEAN) v = L > 0 ? v / (double)L : 0.0;
          o[j] = (float)v;
        }
      }
    }
  }
  if (unpooled_out) {
    for (int64_t i = 0; i < N; ++i) {
      if (rows[inv[i]] < 0) {
        std::memset(unpooled_out + (size_t)i * D, 0, sizeof(float) * D);
        continue;
      }
      const float* e = &t->emb[(size_t)rows[inv[i]] * D];
      std::memcpy(unpooled_out + (size_t)i * D, e, sizeof(float) * D);
    }
  }

  if (uniq_out) std::copy(uniq.begin(), uniq.end(), uniq_out);
  if (rows_out) std::copy(rows.begin(), rows.end(), rows_out);
  if (inv_out) std::copy(inv.begin(), inv.end(), inv_out);
  if (U_out) *U_out = U;
  if (n_new_out) *n_new_out = n_new;

  t->uniq.swap(uniq);
  t->rows.swap(rows);
  t->inv.swap(inv);
  t->bag_offsets.assign(bag_offsets, bag_offsets + (nbags > 0 ? nbags + 1 : 0));
  t->N = N;
  t->B = B;
  t->F = F;
  t->combiner = combiner;
  t->have_batch = true;
  return ORC_OK;
}

// Backward + optimiser.
//  Gradient per unique key (the README's "Reduction" operator; the arithmetic is
//  the chain rule of sum/mean pooling):
//    g(u) = sum over occurrences i with key u of
//           grad_pooled[bag(i)] * (1, or 1/L for mean) + grad_unpooled[i]
//  in double.  Then the optimiser on every touched row (lazy, sparse), in the
//  form of PyTorch's defaults (reading: RecIS is built on the PyTorch
//  ecosystem):
//    Adagrad: acc += g^2;  w -= lr * g / (sqrt(acc) + eps)
//    Adam   : t += 1 (once per call);  m = b1 m + (1-b1) g;  v = b2 v + (1-b2) g^2
//             w -= (lr / (1 - b1^t)) * m / (sqrt(v) / sqrt(1 - b2^t) + eps)
//  Rows touched with zero gradient are still updated (Adam moments decay).
extern "C" int orc_backward_update(orc_table* t, const float* grad_pooled,
                                   const float* grad_unpooled, double* grad_u_out) {
  if (!t || !t->have_batch) return ORC_INVALID_ARG;
  const int D = t->D;
  const int64_t U = (int64_t)t->uniq.size();
  std::vector<double> g((size_t)U * D, 0.0);
  if (grad_pooled) {
    for (int32_t f = 0; f < t->F; ++f) {
      for (int64_t b = 0; b < t->B; ++b) {
        const int64_t bag = (int64_t)f * t->B + b;
        const int64_t lo = t->bag_offsets[bag], hi = t->bag_offsets[bag + 1];
        const float* go = grad_pooled + ((size_t)b * t->F + f) * D;
        const double L = (double)(hi - lo);
        for (int64_t i = lo; i < hi; ++i) {
          double* gu = &g[(size_t)t->inv[i] * D];
          for (int j = 0; j < D; ++j) {
            double term = (double)go[j];
            if (t->combiner == ORC_MEAN) term = term / L;
            gu[j] += term;
          }
        }
      }
    }
  }
  if (grad_unpooled) {
    for (int64_t i = 0; i < t->N; ++i) {
      double* gu = &g[(size_t)t->inv[i] * D];
      const float* gi = grad_unpooled + (size_t)i * D;
      for (int j = 0; j < D; ++j) gu[j] += (double)gi[j];
    }
  }
  if (grad_u_out) std::copy(g.begin(), g.end(), grad_u_out);

  if (t->opt == ORC_ADAM) t->step += 1;
  const double bc1 = 1.0 - std::pow(t->beta1, (double)t->step);
  const double bc2 = 1.0 - std::pow(t->beta2, (double)t->step);
  for (int64_t u = 0; u < U; ++u) {
    const int64_t row = t->rows[u];
    if (row < 0) continue;  // a candidate without a row: its gradient is dropped
    float* w = &t->emb[(size_t)row * D];
    float* st = &t->state[(size_t)row * t->s * D];
    const double* gu = &g[(size_t)u * D];
    for (int j = 0; j < D; ++j) {
      const double gj = gu[j];
      if (t->opt == ORC_ADAGRAD) {
        const double acc = (double)st[j] + gj * gj;
        const double wn = (double)w[j] - t->lr * gj / (std::sqrt(acc) + t->eps);
        st[j] = (float)acc;
        w[j] = (float)wn;
      } else {
        const double m = t->beta1 * (double)st[j] + (1.0 - t->beta1) * gj;
        const double v = t->beta2 * (double)st[D + j] + (1.0 - t->beta2) * gj * gj;
        const double wn =
            (double)w[j] - (t->lr / bc1) * m / (std::sqrt(v) / std::sqrt(bc2) + t->eps);
        st[j] = (float)m;
        st[D + j] = (float)v;
        w[j] = (float)wn;
      }
    }
  }
  return ORC_OK;
}

// live rows: every row that holds a key (freed rows hold -1)
extern "C" int64_t orc_table_size(const orc_table* t) {
  return (int64_t)t->row_key.size() - (int64_t)(t->free_rows.size() - t->free_head);
}
extern "C" int64_t orc_table_step(const orc_table* t) { return t->step; }
extern "C" int64_t orc_table_clock(const orc_table* t) { return t->clock; }

// the live rows in ascending row order (freed rows left out)
extern "C" int orc_table_export(const orc_table* t, int64_t* keys, float* emb, float* state) {
  const int D = t->D, SD = t->s * t->D;
  int64_t k = 0;
  for (size_t row = 0; row < t->row_key.size(); ++row) {
    if (t->row_key[row] == kReserved) continue;
    if (keys) keys[k] = t->row_key[row];
    if (emb) std::copy(&t->emb[row * D], &t->emb[row * D] + D, emb + (size_t)k * D);
    if (state) std::copy(&t->state[row * SD], &t->state[row * SD] + SD, state + (size_t)k * SD);
    ++k;
  }
  return ORC_OK;
}

extern "C" int orc_table_set_admission(orc_table* t, int32_t threshold) {
  if (!t || threshold < 0) return ORC_INVALID_ARG;
  t->admit_threshold = threshold < 1 ? 1 : threshold;
  return ORC_OK;
}

// Eviction: every row, and every candidate, whose last lookup came before
// min_clock is removed; the freed rows join the queue in ascending row order.
extern "C" int orc_table_evict(orc_table* t, int64_t min_clock, int64_t* n_evicted) {
  if (!t) return ORC_INVALID_ARG;
  int64_t n = 0;
  for (size_t row = 0; row < t->row_key.size(); ++row) {
    if (t->row_key[row] == kReserved || t->last_seen[row] >= min_clock) continue;
    t->idmap.erase(t->row_key[row]);
    t->row_key[row] = kReserved;
    t->free_rows.push_back((int64_t)row);
    ++n;
  }
  for (auto it = t->cand.begin(); it != t->cand.end();) {
    if (it->second.second < min_clock) it = t->cand.erase(it);
    else ++it;
  }
  if (n_evicted) *n_evicted = n;
  return ORC_OK;
}

extern "C" int orc_table_import(orc_table* t, int64_t n, const int64_t* keys, const float* emb,
                                const float* state, int64_t step) {
  for (int64_t i = 0; i < n; ++i)
    if (keys[i] == kReserved || t->idmap.count(keys[i])) return ORC_INVALID_ARG;
  const int D = t->D;
  for (int64_t i = 0; i < n; ++i) {
    t->cand.erase(keys[i]);  // an imported key is admitted
    const int64_t row = add_row(t, keys[i]);
    init_row(t, keys[i], row);  // default state when none is given
    std::memcpy(&t->emb[(size_t)row * D], emb + (size_t)i * D, sizeof(float) * D);
    if (state)
      std::memcpy(&t->state[(size_t)row * t->s * D], state + (size_t)i * t->s * D,
                  sizeof(float) * t->s * D);
  }
  t->step = step;
  return ORC_OK;
}

// Table merging (README, Key optimisations > Distributed optimisation >
// parameter aggregation and sharding: "tables of the same attributes --
// dimension, initialiser and so on -- become one logical table when the model
// is created").  Reading: the attributes are all of a table's settings except
// its capacity (dimension, optimiser and its hyper-parameters, initialiser
// scale and seed); a merged table keeps each feature's IDs apart with a tag,
// the feature's rank among the table's features, written above the widest
// value of the table's features.
extern "C" int orc_plan_tables(const orc_feature_attrs* feats, int32_t F, int32_t* table_of,
                               uint64_t* tag_of, int32_t* shift_of, int64_t* table_capacity,
                               int32_t* n_tables) {
  typedef std::tuple<int32_t, int32_t, double, double, double, double, double, double, uint64_t>
      Attrs;
  std::map<Attrs, int32_t> table_id;  // attributes -> logical table
  std::vector<int64_t> members;       // features seen per table
  std::vector<int32_t> widest;        // widest value per table
  std::vector<int64_t> cap;
  for (int32_t f = 0; f < F; ++f) {
    const orc_feature_attrs& a = feats[f];
    if (a.value_bits < 1 || a.value_bits > 62) return ORC_INVALID_ARG;
    const Attrs key(a.dim, a.optimizer, a.lr, a.beta1, a.beta2, a.eps, a.adagrad_init_acc,
                    a.init_scale, a.init_seed);
    auto it = table_id.find(key);
    if (it == table_id.end()) {
      it = table_id.emplace(key, (int32_t)members.size()).first;
      members.push_back(0);
      widest.push_back(0);
      cap.push_back(0);
    }
    const int32_t t = it->second;
    table_of[f] = t;
    tag_of[f] = (uint64_t)members[t];
    members[t] += 1;
    widest[t] = std::max(widest[t], a.value_bits);
    cap[t] += a.capacity;
  }
  for (size_t t = 0; t < members.size(); ++t) {
    // tags 0 .. members-1 need ceil(log2(members)) bits above the values,
    // inside the 63 bits of a non-negative key
    int bits = 0;
    while (((int64_t)1 << bits) < members[t]) ++bits;
    if (widest[t] + bits > 63) return ORC_INVALID_ARG;
    if (table_capacity) table_capacity[t] = cap[t];
  }
  for (int32_t f = 0; f < F; ++f) shift_of[f] = widest[table_of[f]];
  *n_tables = (int32_t)members.size();
  return ORC_OK;
}

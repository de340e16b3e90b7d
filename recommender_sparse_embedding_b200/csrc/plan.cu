// plan.cu -- table merging at model-creation time (RecIS README, Key
// optimisations > Distributed optimisation > parameter aggregation and
// sharding: tables whose attributes -- dimension, initialiser and the like --
// are the same are merged into one logical table when the model is built,
// which cuts the number of lookups and operators).
//
// Host code only.  Features are grouped by their full table attributes
// (everything of recis_table_config except the capacity fields); groups become
// logical tables in order of first appearance, and each feature gets a tag --
// its rank among its table's features -- that keeps its IDs apart from the
// other features' inside the merged table (key = tag << tag_shift | value).
#include <cstring>
#include <vector>

#include "internal.h"

namespace recis {
namespace {

bool same_attrs(const recis_table_config& a, const recis_table_config& b) {
  return a.dim == b.dim && a.optimizer == b.optimizer && a.lr == b.lr && a.beta1 == b.beta1 &&
         a.beta2 == b.beta2 && a.eps == b.eps && a.adagrad_init_acc == b.adagrad_init_acc &&
         a.init_scale == b.init_scale && a.init_seed == b.init_seed;
}

}  // namespace
}  // namespace recis

using namespace recis;

extern "C" recis_status recis_plan_tables(const recis_feature_spec* feats, int32_t F,
                                          int32_t* table_of_feature, uint64_t* tag_of_feature,
                                          int32_t* tag_shift_of_feature,
                                          recis_table_config* tables_out, int32_t* n_tables_out) {
  if (F < 0 || (F > 0 && (!feats || !table_of_feature || !tag_of_feature ||
                          !tag_shift_of_feature || !tables_out)) || !n_tables_out) {
    set_error("plan_tables: bad arguments");
    return RECIS_ERR_INVALID_ARG;
  }
  std::vector<int32_t> first;   // first feature of each table
  std::vector<int64_t> count;   // features per table
  std::vector<int32_t> shift;   // widest value of each table's features
  for (int32_t f = 0; f < F; ++f) {
    const recis_feature_spec& fs = feats[f];
    if (fs.value_bits < 1 || fs.value_bits > 62) {
      set_error("plan_tables: value_bits of feature " + std::to_string(f) + " not in 1..62");
      return RECIS_ERR_INVALID_ARG;
    }
    size_t t = 0;
    while (t < first.size() && !same_attrs(feats[first[t]].table, fs.table)) ++t;
    if (t == first.size()) {
      first.push_back(f);
      count.push_back(0);
      shift.push_back(0);
    }
    table_of_feature[f] = (int32_t)t;
    tag_of_feature[f] = (uint64_t)count[t]++;
    if (fs.value_bits > shift[t]) shift[t] = fs.value_bits;
  }
  for (size_t t = 0; t < first.size(); ++t) {
    // the tags 0 .. count-1 must fit above the values: count <= 2^(63 - shift)
    if (count[t] > ((int64_t)1 << (63 - shift[t]))) {
      set_error("plan_tables: the features of table " + std::to_string(t) +
                " do not fit their tags above " + std::to_string(shift[t]) + "-bit values");
      return RECIS_ERR_INVALID_ARG;
    }
    recis_table_config c = feats[first[t]].table;
    c.initial_capacity = 0;
    c.max_rows = 0;
    bool unbounded = false;
    for (int32_t f = 0; f < F; ++f) {
      if (table_of_feature[f] != (int32_t)t) continue;
      c.initial_capacity += feats[f].table.initial_capacity;
      if (feats[f].table.max_rows <= 0) unbounded = true;
      else c.max_rows += feats[f].table.max_rows;
    }
    if (unbounded) c.max_rows = 0;
    tables_out[t] = c;
  }
  for (int32_t f = 0; f < F; ++f) tag_shift_of_feature[f] = shift[table_of_feature[f]];
  *n_tables_out = (int32_t)first.size();
  return RECIS_OK;
}

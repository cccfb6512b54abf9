// CPU oracle for the dynamic hashed embedding engine.
//
// TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
// bench's CPU-baseline / reference arm load this library.  The product path
// never calls it, and this file shares no code, header, constant table or
// helper with the CUDA library: every formula here is written out again from
// its definition.
//
// What it computes is the plain definition of the method: a dense
// nn.Embedding / EmbeddingBag(mode="sum") over an unbounded table whose rows
// are created on first touch, trained with a sparse (touched-rows-only)
// optimizer.
//
//   * IDMap: std::unordered_map<int64 key, int64 row offset>; the rows live in
//     one std::vector<float> of stride dim * (1 + state arrays).
//     (RecIS overview, "Embedding Engine": a first-level IDMap from feature id
//     to memory offset, a second level of blocks holding the parameters and
//     the optimizer state.)
//   * Multi-table merge: key = table_id << 48 | id, so tables with the same
//     attributes share one map (RecIS overview, "Embedding Engine", multi-table
//     merge).
//   * Offsets of new keys: assigned in the order of a key's first occurrence in
//     the flat batch, continuing from the current row count.  (The pages do
//     not fix an order; this reading makes the key -> row map a function of
//     the key stream.)
//   * Row initialisation: element j of the row of key k is drawn from the
//     splitmix64 stream seeded with k (Steele, Lea, Flood, "Fast splittable
//     pseudorandom number generators", OOPSLA 2014; Vigna's splitmix64.c):
//     z_j = the (j+1)-th output, u = (z_j >> 40) - 2^23, w = u * (0.05 * 2^-23)
//     in fp32, a value in [-0.05, 0.05).  Optimizer state starts at +0.
//   * Forward: pooled[b] = sum over the bag's ids, in fp32, in ascending flat
//     position (nn.Embedding is a row lookup: the background article on RecIS,
//     nn.Embedding section; EmbeddingBag mode="sum": DLRM practice article,
//     section 2.1).
//     EmbeddingBag's other forms (the same practice article names the module,
//     whose "mean" mode and per-sample weights are part of its definition):
//       weighted sum  pooled[b] = sum over i of fl(w_i * W[row_i]), each
//                     product rounded to fp32, added in ascending position;
//       mean          pooled[b] = fl(S_b / len_b), S_b the fp32 in-order sum,
//                     one rounded division; an empty bag gives 0.
//     Mean pooling with per-sample weights is rejected (as in PyTorch).
//   * Backward: for each distinct key k of the batch, g_k = sum over the
//     occurrences of k of grad[bag], accumulated in fp64 in ascending flat
//     position and rounded once to fp32 (sum pooling sends each bag's output
//     gradient to every id in the bag, duplicates counted).  With per-sample
//     weights occurrence i contributes (double)w_i * (double)grad[bag] (an
//     exact product); with mean pooling (double)grad[bag] / (double)len(bag).
//     Then one
//     optimizer step on the touched rows only (DLRM explainer, pitfall 4:
//     sparse optimizer; background article: only row 23 is updated).
//   * Optimizers, elementwise in fp32 with every operation rounded (this file
//     is compiled with -ffp-contract=off):
//       SGD      w = w - lr*g
//       Adagrad  G = G + g*g ; w = w - (lr*g) / (sqrt(G) + eps)
//       Adagrad, row-wise variant: one accumulator per row,
//                G = G + mean_j(g_j^2) (mean in fp64, rounded once);
//                w_j = w_j - (lr*g_j) / (sqrt(G) + eps)
//       Adam     m = b1*m + (1-b1)*g ; v = b2*v + (1-b2)*(g*g)
//                w = w - (lr*(m/bc1)) / (sqrt(v/bc2) + eps),
//                bc1 = 1-b1^t, bc2 = 1-b2^t (t = 1, 2, ... per backward call,
//                computed in fp64 and rounded to fp32; lazy: rows not in the
//                batch keep their m and v).
//
//   * Row storage in bf16 (DLRM practice article, section 4.2: embedding
//     matrices stored in 16-bit floats to halve their bytes), optimizer state
//     in fp32: every stored weight is rounded to the nearest bf16 value, ties
//     to even (the initial row and every optimizer step's result); the
//     forward reads those values and sums in fp32; the optimizer computes in
//     fp32 from them and the fp32 state, then rounds the new weight once.
//
//   * Feature admission and eviction (RecIS overview, code layout: the
//     HashtableHook admission / eviction strategy of the embedding engine;
//     the pages give only its name, so these are the plainest readings):
//       admission  a key gets a row in the first insert call in which its
//                  occurrences over all insert calls so far, this call's
//                  included, reach the threshold (1 = at first sight).  A key
//                  without a row contributes nothing to pooled sums, its
//                  gradients are dropped, and its count is kept.  Keys
//                  admitted in one call get rows in the order of their first
//                  occurrence in that call.
//       eviction   every insert call is one step; a key's stamp is the last
//                  step it occurred in.  evict(max_idle) removes every key
//                  (with or without a row) last seen before step
//                  current - max_idle; their rows become free, and later
//                  admitted keys take free rows in ascending order before new
//                  ones are appended (a reused row starts from the new key's
//                  initial values, state 0).  An evicted key that comes back
//                  is a new key.
//
// A missing key in the backward, or a negative key anywhere, is skipped and
// reported through the return code; the other rows are processed normally.
// A key that is known but not yet admitted is skipped silently.

#include <algorithm>
#include <cmath>
#include <set>
#include <cstdint>
#include <cstring>
#include <unordered_map>
#include <utility>
#include <vector>

namespace {

enum { ORC_OK = 0, ORC_ERR_INVALID = 1, ORC_ERR_NOT_FOUND = 5 };
enum { ORC_SGD = 0, ORC_ADAGRAD = 1, ORC_ADAM = 2, ORC_ADAGRAD_ROWWISE = 3 };

// One step of the splitmix64 generator: the state advances by the golden-ratio
// increment and the output is the state passed through the variant-13 mixer.
uint64_t splitmix64_next(uint64_t* state) {
  *state += 0x9E3779B97F4A7C15ULL;
  uint64_t z = *state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

// Nearest bf16 value of x (the top 16 bits of an fp32 after rounding the low
// 16 bits to nearest, ties to even), returned as the fp32 it widens to.  NaN
// stays a NaN; values past the largest bf16 round to infinity.
float round_bf16(float x) {
  uint32_t u;
  std::memcpy(&u, &x, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) {  // NaN: keep it quiet
    u = (u | 0x00400000u) & 0xffff0000u;
  } else {
    const uint32_t low = u & 0xffffu, half = 0x8000u;
    const uint32_t keep_odd = (u >> 16) & 1u;
    u &= 0xffff0000u;
    if (low > half || (low == half && keep_odd)) u += 0x10000u;  // carries into the exponent as it should
  }
  float y;
  std::memcpy(&y, &u, 4);
  return y;
}

// Initial row of `key`: element j comes from the (j+1)-th output of the
// splitmix64 stream seeded with the key.
void init_row(int64_t key, int dim, float* w) {
  uint64_t s = (uint64_t)key;
  for (int j = 0; j < dim; ++j) {
    uint64_t z = splitmix64_next(&s);
    int32_t u = (int32_t)(z >> 40) - (1 << 23);   // uniform integer in [-2^23, 2^23)
    const float scale = 0.05f * 0x1p-23f;         // exact: 0.05f times a power of two
    w[j] = (float)u * scale;
  }
}

struct Table {
  int dim;
  int opt;
  bool bf16;     // weights stored as bf16 values
  int n_state;   // state floats per row
  float eps, beta1, beta2;
  int64_t adam_t;
  std::unordered_map<int64_t, int64_t> map;
  std::vector<int64_t> key_of_row;  // -1 for a free (evicted) row
  std::vector<float> rows;  // row r at r * stride: dim weights then state
  // admission / eviction
  int64_t admit_threshold = 1;
  bool track = false;                                // stamp keys (needed by evict)
  int64_t step = 0;                                  // insert calls so far
  std::unordered_map<int64_t, int64_t> pending;      // occurrences of keys without a row
  std::unordered_map<int64_t, int64_t> last_seen;    // step of each known key's last occurrence
  std::set<int64_t> free_rows;

  int64_t stride() const { return (int64_t)dim + n_state; }

  float* row(int64_t r) { return rows.data() + r * stride(); }

  int64_t insert_new(int64_t key) {
    int64_t r;
    if (!free_rows.empty()) {  // the smallest free row first
      r = *free_rows.begin();
      free_rows.erase(free_rows.begin());
      key_of_row[r] = key;
    } else {
      r = (int64_t)key_of_row.size();
      key_of_row.push_back(key);
      rows.resize((size_t)(r + 1) * stride(), 0.0f);
    }
    map.emplace(key, r);
    float* w = row(r);
    init_row(key, dim, w);
    for (int j = 0; j < dim; ++j) w[j] = store(w[j]);
    for (int64_t j = dim; j < stride(); ++j) w[j] = 0.0f;
    return r;
  }

  // A weight as the table stores it.
  float store(float v) const { return bf16 ? round_bf16(v) : v; }
};

int state_floats(int opt, int dim) {
  switch (opt) {
    case ORC_SGD: return 0;
    case ORC_ADAGRAD: return dim;
    case ORC_ADAM: return 2 * dim;
    case ORC_ADAGRAD_ROWWISE: return 1;
  }
  return -1;
}

}  // namespace

extern "C" {

uint64_t orc_splitmix64_next(uint64_t* state) { return splitmix64_next(state); }

void orc_init_row(int64_t key, int dim, float* out) { init_row(key, dim, out); }

// key = table_id << 48 | id  (id < 2^48, 0 <= table_id < 2^15)
int orc_pack_keys(const int32_t* table_ids, const int64_t* ids, int64_t n, int64_t* keys) {
  int rc = ORC_OK;
  for (int64_t i = 0; i < n; ++i) {
    int64_t t = table_ids[i], id = ids[i];
    if (t < 0 || t >= (1 << 15) || id < 0 || id >= (int64_t(1) << 48)) {
      keys[i] = -1;
      rc = ORC_ERR_INVALID;
      continue;
    }
    keys[i] = (t << 48) | id;
  }
  return rc;
}

// storage: 0 fp32 weights, 1 bf16 weights (state fp32 either way)
void* orc_create_ex(int dim, int opt, float eps, float beta1, float beta2, int storage) {
  if (dim <= 0 || state_floats(opt, dim) < 0 || storage < 0 || storage > 1) return nullptr;
  Table* t = new Table();
  t->dim = dim;
  t->opt = opt;
  t->bf16 = storage == 1;
  t->n_state = state_floats(opt, dim);
  t->eps = eps;
  t->beta1 = beta1;
  t->beta2 = beta2;
  t->adam_t = 0;
  return t;
}

void* orc_create(int dim, int opt, float eps, float beta1, float beta2) {
  return orc_create_ex(dim, opt, eps, beta1, beta2, 0);
}

float orc_round_bf16(float x) { return round_bf16(x); }

void orc_destroy(void* h) { delete (Table*)h; }

int64_t orc_size(void* h) { return (int64_t)((Table*)h)->key_of_row.size(); }

int64_t orc_stride(void* h) { return ((Table*)h)->stride(); }

// One insert call (lookup_or_insert, forward).  Without admission (threshold
// 1) this is: sequential in i, a key not yet in the map gets the next row.
// With admission: the call's occurrences of each key without a row are added
// to its count first; keys whose count reaches the threshold are admitted in
// the order of their first occurrence in the call; then every position's row
// is read (-1 for a key still without a row).
int orc_lookup_or_insert(void* h, const int64_t* keys, int64_t n, int64_t* offsets_out) {
  Table* t = (Table*)h;
  int rc = ORC_OK;
  t->step += 1;
  std::vector<int64_t> first;  // keys without a row, by first occurrence in the call
  std::unordered_map<int64_t, int64_t> here;
  for (int64_t i = 0; i < n; ++i) {
    const int64_t k = keys[i];
    if (k < 0) {
      rc = ORC_ERR_INVALID;
      continue;
    }
    if (t->track) t->last_seen[k] = t->step;
    if (t->map.count(k)) continue;
    if (here[k]++ == 0) first.push_back(k);
  }
  for (int64_t k : first) {
    const int64_t total = t->pending[k] + here[k];
    if (total >= t->admit_threshold) {
      t->pending.erase(k);
      t->insert_new(k);
    } else {
      t->pending[k] = total;
    }
  }
  for (int64_t i = 0; i < n; ++i) {
    const int64_t k = keys[i];
    auto it = k < 0 ? t->map.end() : t->map.find(k);
    if (offsets_out) offsets_out[i] = it == t->map.end() ? -1 : it->second;
  }
  return rc;
}

// Admission threshold (occurrences before a key gets a row; <= 1: at once)
// and access tracking (stamps for evict); set before the first insert call.
void orc_set_hooks(void* h, int64_t threshold, int track) {
  Table* t = (Table*)h;
  t->admit_threshold = std::max<int64_t>(1, threshold);
  t->track = track != 0;
}

// Evict every key last seen before step (current - max_idle); returns the
// number of rows freed.
int64_t orc_evict(void* h, int64_t max_idle) {
  Table* t = (Table*)h;
  const int64_t keep_from = t->step - max_idle;
  int64_t freed = 0;
  std::vector<int64_t> gone;
  for (const auto& kv : t->last_seen)
    if (kv.second < keep_from) gone.push_back(kv.first);
  for (int64_t k : gone) {
    t->last_seen.erase(k);
    t->pending.erase(k);
    auto it = t->map.find(k);
    if (it != t->map.end()) {
      t->key_of_row[it->second] = -1;
      t->free_rows.insert(it->second);
      t->map.erase(it);
      ++freed;
    }
  }
  return freed;
}

// Keys with a row.
int64_t orc_live(void* h) { return (int64_t)((Table*)h)->map.size(); }

// Read-only lookup: -1 where the key is absent.
void orc_lookup(void* h, const int64_t* keys, int64_t n, int64_t* offsets_out) {
  Table* t = (Table*)h;
  for (int64_t i = 0; i < n; ++i) {
    auto it = t->map.find(keys[i]);
    offsets_out[i] = it == t->map.end() ? -1 : it->second;
  }
}

// mode: 0 sum, 1 mean.  psw: per-sample weights float[n] or null.
int orc_forward_ex(void* h, const int64_t* keys, const int64_t* bag_offsets, int64_t n_bags,
                   const float* psw, int mode, float* pooled) {
  Table* t = (Table*)h;
  if (mode != 0 && mode != 1) return ORC_ERR_INVALID;
  if (mode == 1 && psw) return ORC_ERR_INVALID;
  int64_t n = n_bags > 0 ? bag_offsets[n_bags] : 0;
  std::vector<int64_t> off(n);
  int rc = orc_lookup_or_insert(h, keys, n, off.data());
  for (int64_t b = 0; b < n_bags; ++b) {
    float* out = pooled + b * t->dim;
    for (int j = 0; j < t->dim; ++j) out[j] = 0.0f;
    for (int64_t i = bag_offsets[b]; i < bag_offsets[b + 1]; ++i) {
      if (off[i] < 0) continue;
      const float* w = t->row(off[i]);
      if (psw) {
        for (int j = 0; j < t->dim; ++j) {
          const float prod = psw[i] * w[j];
          out[j] = out[j] + prod;
        }
      } else {
        for (int j = 0; j < t->dim; ++j) out[j] = out[j] + w[j];
      }
    }
    const int64_t len = bag_offsets[b + 1] - bag_offsets[b];
    if (mode == 1 && len > 0)
      for (int j = 0; j < t->dim; ++j) out[j] = out[j] / (float)len;
  }
  return rc;
}

int orc_forward(void* h, const int64_t* keys, const int64_t* bag_offsets, int64_t n_bags,
                float* pooled) {
  return orc_forward_ex(h, keys, bag_offsets, n_bags, nullptr, 0, pooled);
}

int orc_backward_update_ex(void* h, const int64_t* keys, const int64_t* bag_offsets, int64_t n_bags,
                           const float* psw, int mode, const float* grad, float lr) {
  Table* t = (Table*)h;
  const int d = t->dim;
  if (mode != 0 && mode != 1) return ORC_ERR_INVALID;
  if (mode == 1 && psw) return ORC_ERR_INVALID;
  int rc = ORC_OK;
  int64_t n = n_bags > 0 ? bag_offsets[n_bags] : 0;
  t->adam_t += 1;

  // (key, flat position, bag) of every valid occurrence, sorted by key then position
  struct Occ { int64_t key, pos, bag; };
  std::vector<Occ> occ;
  occ.reserve(n);
  for (int64_t b = 0; b < n_bags; ++b)
    for (int64_t i = bag_offsets[b]; i < bag_offsets[b + 1]; ++i) {
      int64_t k = keys[i];
      if (k < 0) { rc = ORC_ERR_INVALID; continue; }
      if (t->map.find(k) == t->map.end()) {
        if (!t->pending.count(k)) rc = rc ? rc : ORC_ERR_NOT_FOUND;  // a key not admitted yet: skipped
        continue;
      }
      occ.push_back({k, i, b});
    }
  std::sort(occ.begin(), occ.end(), [](const Occ& a, const Occ& b) {
    return a.key != b.key ? a.key < b.key : a.pos < b.pos;
  });

  // Adam bias corrections for this step, in fp64, rounded once
  const float b1 = t->beta1, b2 = t->beta2;
  const float c1 = (float)(1.0 - (double)b1), c2 = (float)(1.0 - (double)b2);
  const float bc1 = (float)(1.0 - std::pow((double)b1, (double)t->adam_t));
  const float bc2 = (float)(1.0 - std::pow((double)b2, (double)t->adam_t));

  std::vector<double> acc(d);
  std::vector<float> g(d);
  size_t a = 0;
  while (a < occ.size()) {
    size_t e = a;
    while (e < occ.size() && occ[e].key == occ[a].key) ++e;
    std::fill(acc.begin(), acc.end(), 0.0);
    for (size_t q = a; q < e; ++q) {
      const float* gb = grad + occ[q].bag * d;
      if (psw) {
        const double wq = (double)psw[occ[q].pos];
        for (int j = 0; j < d; ++j) acc[j] += wq * (double)gb[j];
      } else if (mode == 1) {
        const double len = (double)(bag_offsets[occ[q].bag + 1] - bag_offsets[occ[q].bag]);
        for (int j = 0; j < d; ++j) acc[j] += (double)gb[j] / len;
      } else {
        for (int j = 0; j < d; ++j) acc[j] += (double)gb[j];
      }
    }
    for (int j = 0; j < d; ++j) g[j] = (float)acc[j];

    float* w = t->row(t->map[occ[a].key]);
    switch (t->opt) {
      case ORC_SGD:
        for (int j = 0; j < d; ++j) w[j] = t->store(w[j] - lr * g[j]);
        break;
      case ORC_ADAGRAD: {
        float* G = w + d;
        for (int j = 0; j < d; ++j) {
          G[j] = G[j] + g[j] * g[j];
          w[j] = t->store(w[j] - (lr * g[j]) / (std::sqrt(G[j]) + t->eps));
        }
        break;
      }
      case ORC_ADAGRAD_ROWWISE: {
        double ss = 0.0;
        for (int j = 0; j < d; ++j) ss += (double)g[j] * (double)g[j];
        float* G = w + d;
        G[0] = G[0] + (float)(ss / d);
        float den = std::sqrt(G[0]) + t->eps;
        for (int j = 0; j < d; ++j) w[j] = t->store(w[j] - (lr * g[j]) / den);
        break;
      }
      case ORC_ADAM: {
        float* m = w + d;
        float* v = w + 2 * d;
        for (int j = 0; j < d; ++j) {
          m[j] = b1 * m[j] + c1 * g[j];
          v[j] = b2 * v[j] + c2 * (g[j] * g[j]);
          float mhat = m[j] / bc1;
          float vhat = v[j] / bc2;
          w[j] = t->store(w[j] - (lr * mhat) / (std::sqrt(vhat) + t->eps));
        }
        break;
      }
    }
    a = e;
  }
  return rc;
}

int orc_backward_update(void* h, const int64_t* keys, const int64_t* bag_offsets, int64_t n_bags,
                        const float* grad, float lr) {
  return orc_backward_update_ex(h, keys, bag_offsets, n_bags, nullptr, 0, grad, lr);
}

// Export in row-offset order: keys[r] is the key whose offset is r; rows holds
// stride floats per row (weights then state).  Any pointer may be null.
void orc_export(void* h, int64_t* keys, float* rows) {
  Table* t = (Table*)h;
  int64_t n = (int64_t)t->key_of_row.size();
  if (keys) std::memcpy(keys, t->key_of_row.data(), sizeof(int64_t) * n);
  if (rows) std::memcpy(rows, t->rows.data(), sizeof(float) * n * t->stride());
}

// Overwrite the first n rows (stride floats each, weights then state) with
// the given values, as stored (no rounding): lets a test start a step from
// rows taken from another table.
void orc_import_rows(void* h, const float* rows, int64_t n) {
  Table* t = (Table*)h;
  const int64_t m = std::min<int64_t>(n, (int64_t)t->key_of_row.size());
  std::memcpy(t->rows.data(), rows, sizeof(float) * m * t->stride());
}

// Rows (weights then state) of the given keys; absent keys give NaN rows and
// offset -1.  Returns the number of absent keys.
int64_t orc_get_rows(void* h, const int64_t* keys, int64_t n, float* rows_out) {
  Table* t = (Table*)h;
  int64_t missing = 0;
  const int64_t s = t->stride();
  for (int64_t i = 0; i < n; ++i) {
    auto it = t->map.find(keys[i]);
    if (it == t->map.end()) {
      for (int64_t j = 0; j < s; ++j) rows_out[i * s + j] = std::nanf("");
      ++missing;
      continue;
    }
    std::memcpy(rows_out + i * s, t->row(it->second), sizeof(float) * s);
  }
  return missing;
}

}  // extern "C"

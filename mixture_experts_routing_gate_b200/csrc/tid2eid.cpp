// Host-side greedy tid2eid builder ("How was DeepSeek V4's tid2eid derived?", greedy rule under
// eq. 2): tokens in descending frequency each take the k experts of least current load, which then
// carry p_i / k more.  Experts are kept in an ordered set keyed by (load, expert index), so the k
// lightest are the first k entries and equal loads resolve to the lower index; each step costs
// O(k log n) instead of a full sort of the loads.
//
// The randomised variant (same page, the paragraph after the reference implementation) visits the
// tokens in caller-given orders instead, builds one table per order, and keeps a table of least
// max_vio = n * max_e f_e - 1.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <numeric>
#include <set>
#include <utility>
#include <vector>

#include "../../include/moe.h"

namespace {

// One greedy pass over `order` (token ids); fills table [m, k] and f [n].
void greedy(const double* p, const int* order, int m, int n_experts, int k, int32_t* table, std::vector<double>& f) {
  f.assign(n_experts, 0.0);
  std::set<std::pair<double, int>> by_load;
  for (int j = 0; j < n_experts; ++j) by_load.emplace(0.0, j);
  std::vector<int> picked(k);
  for (int v = 0; v < m; ++v) {
    const int i = order[v];
    auto it = by_load.begin();
    for (int j = 0; j < k; ++j, ++it) picked[j] = it->second;
    by_load.erase(by_load.begin(), it);
    const double q = p[i] / k;
    int32_t* row = table + static_cast<size_t>(i) * k;
    for (int j = 0; j < k; ++j) {
      const int e = picked[j];
      row[j] = e;
      f[e] += q;
      by_load.emplace(f[e], e);
    }
  }
}

bool valid_frequencies(const double* p, int m) {
  for (int i = 0; i < m; ++i)
    if (!std::isfinite(p[i]) || p[i] < 0.0) return false;
  return true;
}

double max_vio(const std::vector<double>& f) {
  const double mx = *std::max_element(f.begin(), f.end());
  const double scaled = mx * static_cast<double>(f.size());
  return scaled - 1.0;
}

}  // namespace

extern "C" moe_status moe_build_tid2eid(const double* p, int m, int n_experts, int k, int32_t* tid2eid,
                                        double* loads) {
  if (m < 0 || n_experts < 1 || k < 1 || k > n_experts) return MOE_ERR_INVALID;
  if (m > 0 && (p == nullptr || tid2eid == nullptr)) return MOE_ERR_INVALID;
  if (!valid_frequencies(p, m)) return MOE_ERR_INVALID;

  std::vector<int> order(m);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [p](int a, int b) { return p[a] > p[b]; });

  std::vector<double> f;
  greedy(p, order.data(), m, n_experts, k, tid2eid, f);
  if (loads != nullptr) std::copy(f.begin(), f.end(), loads);
  return MOE_OK;
}

extern "C" moe_status moe_build_tid2eid_best(const double* p, int m, int n_experts, int k, const int32_t* orders,
                                             int runs, int32_t* tid2eid, double* loads, double* max_vio_out,
                                             int32_t* kept) {
  if (m < 0 || n_experts < 1 || k < 1 || k > n_experts || runs < 1) return MOE_ERR_INVALID;
  if (orders == nullptr || (m > 0 && (p == nullptr || tid2eid == nullptr))) return MOE_ERR_INVALID;
  if (!valid_frequencies(p, m)) return MOE_ERR_INVALID;
  // every order must visit each token exactly once
  std::vector<char> seen(m);
  for (int r = 0; r < runs; ++r) {
    std::fill(seen.begin(), seen.end(), 0);
    const int32_t* o = orders + static_cast<size_t>(r) * m;
    for (int v = 0; v < m; ++v) {
      if (o[v] < 0 || o[v] >= m || seen[o[v]]) return MOE_ERR_INVALID;
      seen[o[v]] = 1;
    }
  }

  std::vector<int32_t> table(static_cast<size_t>(m) * k);
  std::vector<double> f;
  double best = 0.0;
  int best_run = -1;
  for (int r = 0; r < runs; ++r) {
    const int32_t* o = orders + static_cast<size_t>(r) * m;
    greedy(p, o, m, n_experts, k, table.data(), f);
    const double vio = max_vio(f);
    if (max_vio_out != nullptr) max_vio_out[r] = vio;
    if (best_run < 0 || vio < best) {  // equal max_vio: the earlier run stays
      best = vio;
      best_run = r;
      std::copy(table.begin(), table.end(), tid2eid);
      if (loads != nullptr) std::copy(f.begin(), f.end(), loads);
    }
  }
  if (kept != nullptr) *kept = best_run;
  return MOE_OK;
}

// ------------------------------------------------------------------------------------------------
// tables on disk: "MOETID01", int32 m, k, n_experts, 0, uint64 FNV-1a of p's bytes, int32 ids
// ------------------------------------------------------------------------------------------------
namespace {

constexpr char kMagic[8] = {'M', 'O', 'E', 'T', 'I', 'D', '0', '1'};

struct TableHeader {
  char magic[8];
  int32_t m, k, n_experts, reserved;
  uint64_t p_hash;
};
static_assert(sizeof(TableHeader) == 32, "file header layout");

// FNV-1a, 64-bit, over the bytes of the m fp64 frequencies.
uint64_t hash_of(const double* p, int m) {
  uint64_t h = 14695981039346656037ull;
  const unsigned char* b = reinterpret_cast<const unsigned char*>(p);
  for (size_t i = 0; i < static_cast<size_t>(m) * sizeof(double); ++i) {
    h ^= b[i];
    h *= 1099511628211ull;
  }
  return h;
}

bool ids_in_range(const int32_t* t, size_t count, int n_experts) {
  for (size_t i = 0; i < count; ++i)
    if (t[i] < 0 || t[i] >= n_experts) return false;
  return true;
}

struct File {
  FILE* f;
  explicit File(FILE* f_) : f(f_) {}
  ~File() {
    if (f != nullptr) fclose(f);
  }
};

moe_status read_header(FILE* f, TableHeader* h) {
  if (fread(h, sizeof(*h), 1, f) != 1) return ferror(f) ? MOE_ERR_IO : MOE_ERR_INVALID;
  if (memcmp(h->magic, kMagic, sizeof(kMagic)) != 0 || h->m < 0 || h->k < 1 || h->n_experts < 1 ||
      h->k > h->n_experts)
    return MOE_ERR_INVALID;
  return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_tid2eid_save(const char* path, const int32_t* tid2eid, int m, int k, int n_experts,
                                       const double* p) {
  if (path == nullptr || m < 0 || k < 1 || n_experts < 1 || k > n_experts) return MOE_ERR_INVALID;
  if (m > 0 && tid2eid == nullptr) return MOE_ERR_INVALID;
  const size_t count = static_cast<size_t>(m) * k;
  if (!ids_in_range(tid2eid, count, n_experts)) return MOE_ERR_INVALID;
  if (p != nullptr && !valid_frequencies(p, m)) return MOE_ERR_INVALID;
  TableHeader h;
  memcpy(h.magic, kMagic, sizeof(kMagic));
  h.m = m;
  h.k = k;
  h.n_experts = n_experts;
  h.reserved = 0;
  h.p_hash = p != nullptr ? hash_of(p, m) : 0;
  File file(fopen(path, "wb"));
  if (file.f == nullptr) return MOE_ERR_IO;
  if (fwrite(&h, sizeof(h), 1, file.f) != 1) return MOE_ERR_IO;
  if (count > 0 && fwrite(tid2eid, sizeof(int32_t), count, file.f) != count) return MOE_ERR_IO;
  FILE* f = file.f;
  file.f = nullptr;
  return fclose(f) == 0 ? MOE_OK : MOE_ERR_IO;
}

extern "C" moe_status moe_tid2eid_header(const char* path, int* m, int* k, int* n_experts) {
  if (path == nullptr || m == nullptr || k == nullptr || n_experts == nullptr) return MOE_ERR_INVALID;
  File file(fopen(path, "rb"));
  if (file.f == nullptr) return MOE_ERR_IO;
  TableHeader h;
  const moe_status st = read_header(file.f, &h);
  if (st != MOE_OK) return st;
  *m = h.m;
  *k = h.k;
  *n_experts = h.n_experts;
  return MOE_OK;
}

extern "C" moe_status moe_tid2eid_load(const char* path, int32_t* tid2eid, int m, int k, int n_experts,
                                       const double* p) {
  if (path == nullptr || m < 0 || k < 1 || n_experts < 1 || k > n_experts) return MOE_ERR_INVALID;
  if (m > 0 && tid2eid == nullptr) return MOE_ERR_INVALID;
  File file(fopen(path, "rb"));
  if (file.f == nullptr) return MOE_ERR_IO;
  TableHeader h;
  const moe_status st = read_header(file.f, &h);
  if (st != MOE_OK) return st;
  if (h.m != m || h.k != k || h.n_experts != n_experts) return MOE_ERR_INVALID;
  if (p != nullptr && h.p_hash != hash_of(p, m)) return MOE_ERR_INVALID;
  const size_t count = static_cast<size_t>(m) * k;
  // read into a buffer of our own: the caller's table is written only once every check has passed
  std::vector<int32_t> ids(count);
  if (count > 0 && fread(ids.data(), sizeof(int32_t), count, file.f) != count)
    return ferror(file.f) ? MOE_ERR_IO : MOE_ERR_INVALID;
  if (fgetc(file.f) != EOF) return MOE_ERR_INVALID;   // trailing bytes: not a table of this size
  if (!ids_in_range(ids.data(), count, n_experts)) return MOE_ERR_INVALID;
  if (count > 0) memcpy(tid2eid, ids.data(), count * sizeof(int32_t));
  return MOE_OK;
}

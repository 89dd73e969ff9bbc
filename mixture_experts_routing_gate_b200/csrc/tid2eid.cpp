// Host-side greedy tid2eid builder ("How was DeepSeek V4's tid2eid derived?", greedy rule under
// eq. 2): tokens in descending frequency each take the k experts of least current load, which then
// carry p_i / k more.  Experts are kept in an ordered set keyed by (load, expert index), so the k
// lightest are the first k entries and equal loads resolve to the lower index; each step costs
// O(k log n) instead of a full sort of the loads.
#include <algorithm>
#include <cmath>
#include <numeric>
#include <set>
#include <utility>
#include <vector>

#include "../../include/moe.h"

extern "C" moe_status moe_build_tid2eid(const double* p, int m, int n_experts, int k, int32_t* tid2eid,
                                        double* loads) {
  if (m < 0 || n_experts < 1 || k < 1 || k > n_experts) return MOE_ERR_INVALID;
  if (m > 0 && (p == nullptr || tid2eid == nullptr)) return MOE_ERR_INVALID;
  for (int i = 0; i < m; ++i)
    if (!std::isfinite(p[i]) || p[i] < 0.0) return MOE_ERR_INVALID;

  std::vector<int> order(m);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [p](int a, int b) { return p[a] > p[b]; });

  std::vector<double> f(n_experts, 0.0);
  std::set<std::pair<double, int>> by_load;
  for (int j = 0; j < n_experts; ++j) by_load.emplace(0.0, j);

  std::vector<int> picked(k);
  for (const int i : order) {
    auto it = by_load.begin();
    for (int j = 0; j < k; ++j, ++it) picked[j] = it->second;
    by_load.erase(by_load.begin(), it);
    const double q = p[i] / k;
    int32_t* row = tid2eid + static_cast<size_t>(i) * k;
    for (int j = 0; j < k; ++j) {
      const int e = picked[j];
      row[j] = e;
      f[e] += q;
      by_load.emplace(f[e], e);
    }
  }
  if (loads != nullptr) std::copy(f.begin(), f.end(), loads);
  return MOE_OK;
}

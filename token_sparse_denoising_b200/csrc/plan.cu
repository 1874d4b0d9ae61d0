// plan.cu -- hsa_plan_groups: the schedule of a whole HSA run, on the host.
//
// HSA summary §2.1: N tokens split into K disjoint groups G_1..G_K; group k gets
// a step budget s_k that divides T, the baseline group has s_1 = T, and group k
// runs at global iteration i when i mod (T/s_k) = 0.  §2.4: the first and last
// m iterations run every token.  Iterations are 0-based (step i moves sigma_i
// to sigma_{i+1}), so the rule alone fires exactly s_k times per run.
#include <string>

#include "common.cuh"

extern "C" int hsa_plan_groups(int T, int K, const int* h_budgets, const int* h_group_sizes, int N, int m,
                               int sigma_kind, float shift, float* h_sigmas, uint8_t* h_active_tab,
                               int* h_n_active) {
  using hsa::set_error;
  if (T <= 0 || K <= 0 || !h_budgets || !h_group_sizes || N < 0)
    return set_error(HSA_EINVAL, "plan: need T > 0, K > 0, budgets and group sizes");
  if (h_budgets[0] != T) return set_error(HSA_EINVAL, "plan: the baseline group must have s_1 = T");
  long long total = 0;
  for (int k = 0; k < K; ++k) {
    const int s = h_budgets[k];
    if (s <= 0 || T % s != 0)
      return set_error(HSA_EINVAL, "plan: budget s_" + std::to_string(k + 1) + " does not divide T");
    if (k > 0 && s > h_budgets[k - 1]) return set_error(HSA_EINVAL, "plan: budgets must be non-increasing");
    if (h_group_sizes[k] < 0) return set_error(HSA_EINVAL, "plan: negative group size");
    total += h_group_sizes[k];
  }
  if (total != N) return set_error(HSA_EINVAL, "plan: group sizes must sum to N");
  if (m < 0 || 2 * m > T) return set_error(HSA_EINVAL, "plan: need 0 <= 2m <= T");
  if (sigma_kind != 0 && sigma_kind != 1) return set_error(HSA_EINVAL, "plan: sigma_kind must be 0 or 1");
  if (sigma_kind == 1 && !(shift > 0.0f)) return set_error(HSA_EINVAL, "plan: shift must be positive");

  if (h_sigmas) {
    for (int i = 0; i <= T; ++i) {
      double sig = 1.0 - static_cast<double>(i) / static_cast<double>(T);
      if (sigma_kind == 1) {
        const double s = static_cast<double>(shift);
        sig = s * sig / (1.0 + (s - 1.0) * sig);
      }
      h_sigmas[i] = static_cast<float>(sig);
    }
  }
  for (int i = 0; i < T; ++i) {
    const bool window_full = i < m || i >= T - m;
    long long active = 0;
    for (int k = 0; k < K; ++k) {
      const int period = T / h_budgets[k];
      const bool on = window_full || (i % period == 0);
      if (h_active_tab) h_active_tab[static_cast<size_t>(i) * K + k] = on ? 1 : 0;
      if (on) active += h_group_sizes[k];
    }
    if (h_n_active) h_n_active[i] = static_cast<int>(active);
  }
  return HSA_OK;
}

// Greedy mixed-precision layer allocation (host): layers move from the lower
// to the higher-bit format in order of error reduction per added byte while
// the byte budget allows ("AngelSlim Shrinks ..." bullet list;
// lemmy.durstig.online post 66506, "Full-Hessian scoring").
//
// IEEE fp64 throughout, fixed evaluation order, compiled with
// -ffp-contract=off: the picks depend on the inputs alone.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <numeric>
#include <vector>

#include "../../include/stq1.h"

extern "C" int stq1_mix_allocate(const double* err_low, const double* err_high, const double* bytes_low,
                                 const double* bytes_high, int64_t n_layers, double budget, uint8_t* pick) {
  if (!err_low || !err_high || !bytes_low || !bytes_high || !pick) return STQ1_ERR_NULL;
  if (n_layers <= 0) return STQ1_ERR_SHAPE;
  if (!std::isfinite(budget)) return STQ1_ERR_VALUE;
  const size_t n = static_cast<size_t>(n_layers);
  std::vector<double> gain(n);
  for (size_t i = 0; i < n; ++i) {
    if (!std::isfinite(err_low[i]) || !std::isfinite(err_high[i]) || !std::isfinite(bytes_low[i]) ||
        !std::isfinite(bytes_high[i]) || !(bytes_high[i] > bytes_low[i]))
      return STQ1_ERR_VALUE;
    gain[i] = (err_low[i] - err_high[i]) / (bytes_high[i] - bytes_low[i]);
    if (!std::isfinite(gain[i])) return STQ1_ERR_VALUE;
  }
  std::vector<size_t> order(n);
  std::iota(order.begin(), order.end(), size_t{0});
  std::sort(order.begin(), order.end(), [&](size_t a, size_t b) {
    return gain[a] > gain[b] || (gain[a] == gain[b] && a < b);
  });
  double total = 0.0;
  for (size_t i = 0; i < n; ++i) total += bytes_low[i];
  for (size_t i = 0; i < n; ++i) pick[i] = 0;
  for (size_t r = 0; r < n; ++r) {
    const size_t i = order[r];
    if (gain[i] <= 0.0) break;
    const double cost = bytes_high[i] - bytes_low[i];
    if (total + cost <= budget) {
      pick[i] = 1;
      total += cost;
    }
  }
  return STQ1_OK;
}

// sq_alloc.cu -- offline unit bit-width allocation of libsq (host code; no GPU work).
//
// STEPQuant explainer, lifetime-aware allocation paragraph: under a fixed average bit budget,
// units whose error is large and long-lived get more bits; the width of each unit (a whole head,
// or one key row) is chosen from a score that combines its reconstruction distortion with how
// long, on average, its memory persists; a few high-risk units stay FP16 as pivots. The
// Block-GTQ page describes the allocation rule used here: repeatedly give the next bits to the
// unit whose error they reduce most, which is optimal under the integer constraint for a
// separable objective.
//
// Reading. Unit u has the variance var_u of its state entries and the mean lifetime L_u of its
// memory (1 / (1 - mean gate) for a gate that keeps a fraction alpha per step). Its risk is
// R_u = L_u var_u, and at b bits its score is R_u 2^(-2b) (the distortion of a uniform b-bit
// quantizer scales as var 2^(-2b)). The n_pivots units of largest risk (ties: lower index) are
// FP16 pivots (width 16). Every other unit starts at 2 bits; the budget adds K steps of 2 bits,
// K = floor((avg_bits - 2) n' / 2) for the n' non-pivot units (at most 3 per unit: widths
// 2, 4, 6, 8); each step goes to the unit with the largest score reduction
// R_u (2^(-2b_u) - 2^(-2b_u - 4)) (ties: lower index). Each unit's reductions shrink by 16x per
// step, so this greedy choice minimizes the total score sum_u R_u 2^(-2 b_u).
#include <math.h>

#include <algorithm>
#include <queue>
#include <vector>

#include "sq.h"

extern "C" sq_status sq_allocate_bits(int32_t n_units, const float* variance,
                                      const float* lifetime, float avg_bits, int32_t n_pivots,
                                      uint8_t* bits_map, uint8_t* pivot_mask) {
  if (n_units < 1 || !variance || !lifetime || !bits_map) return SQ_ERR_INVALID_ARG;
  if (n_pivots < 0 || n_pivots >= n_units) return SQ_ERR_INVALID_ARG;
  if (!(avg_bits >= 2.0f && avg_bits <= 8.0f)) return SQ_ERR_INVALID_ARG;
  std::vector<double> risk((size_t)n_units);
  for (int32_t u = 0; u < n_units; ++u) {
    const float v = variance[u], l = lifetime[u];
    if (!(v >= 0.0f) || !(l >= 0.0f) || !isfinite(v) || !isfinite(l)) return SQ_ERR_INVALID_ARG;
    risk[(size_t)u] = (double)v * (double)l;
  }
  // pivots: the largest risks, ties to the lower index
  std::vector<int32_t> order((size_t)n_units);
  for (int32_t u = 0; u < n_units; ++u) order[(size_t)u] = u;
  std::stable_sort(order.begin(), order.end(),
                   [&](int32_t a, int32_t b) { return risk[(size_t)a] > risk[(size_t)b]; });
  std::vector<uint8_t> width((size_t)n_units, 2);
  for (int32_t p = 0; p < n_pivots; ++p) width[(size_t)order[(size_t)p]] = 16;
  const int32_t n_q = n_units - n_pivots;
  long long steps = (long long)floor(((double)avg_bits - 2.0) * (double)n_q / 2.0 + 1e-9);
  if (steps < 0) steps = 0;
  if (steps > 3LL * n_q) steps = 3LL * n_q;
  // greedy: the largest score reduction first; the heap key is R_u 2^(-2b_u), the common factor
  // 15/16 left out; ties to the lower index
  struct Item {
    double gain;
    int32_t u;
  };
  auto cmp = [](const Item& a, const Item& b) {
    return a.gain < b.gain || (a.gain == b.gain && a.u > b.u);
  };
  std::priority_queue<Item, std::vector<Item>, decltype(cmp)> heap(cmp);
  for (int32_t u = 0; u < n_units; ++u)
    if (width[(size_t)u] != 16) heap.push({ldexp(risk[(size_t)u], -4), u});
  for (long long s = 0; s < steps && !heap.empty(); ++s) {
    const Item it = heap.top();
    heap.pop();
    uint8_t& w = width[(size_t)it.u];
    w = (uint8_t)(w + 2);
    if (w < 8) heap.push({ldexp(risk[(size_t)it.u], -2 * (int)w), it.u});
  }
  for (int32_t u = 0; u < n_units; ++u) {
    bits_map[u] = width[(size_t)u];
    if (pivot_mask) pivot_mask[u] = width[(size_t)u] == 16 ? 1 : 0;
  }
  return SQ_OK;
}

// Cost-aware tree sizing (EAGLE-4 write-up, "Деревья проверки EAGLE-4 и
// утилита управления"): a latency table measured once on the GPU, and the
// per-level decision that weighs a level's gain in cumulative probability
// against its marginal verification cost.  Host code only: the decision sits
// between two draft-model levels, where the host drives the draft loop; the
// gains come from eagle_tree_grow_gains.
//
//   cost     multilinear interpolation of us[B][L][N] over the ascending grids,
//            the end segments extended outside them, a single-point axis
//            constant;
//   level l  grows the verified set from (l-1)k to lk candidates per
//            sequence; ratio = (sum of the batch's gains) / (C(lk) - C((l-1)k))
//            in tokens per unit of cost (infinite when the cost does not
//            grow); the level is kept iff ratio >= threshold;
//   width    (widening or deepening) the level's candidates one at a time in
//            descending V, the j-th best of every sequence together: gain =
//            sum over the batch of its V, marginal cost C(n + j) - C(n + j - 1)
//            with n candidates per sequence chosen before this level; taken
//            while gain > 0 and gain / cost >= threshold (a cost that does not
//            grow passes); the number taken is the level's width.
#include <cmath>

#include "eagle_internal.h"

namespace {

bool valid_axis(const double* g, int n) {
  if (!g || n < 1) return false;
  for (int i = 0; i < n; ++i)
    if (!std::isfinite(g[i]) || (i > 0 && !(g[i] > g[i - 1]))) return false;
  return true;
}

bool valid_table(const eagle_cost_table_t* t) {
  if (!t || !t->us || !valid_axis(t->B, t->nB) || !valid_axis(t->L, t->nL) || !valid_axis(t->N, t->nN)) return false;
  const long long cells = (long long)t->nB * t->nL * t->nN;
  for (long long i = 0; i < cells; ++i)
    if (!std::isfinite(t->us[i])) return false;
  return true;
}

// Lower grid index and the upper point's weight for x.
void axis_pos(const double* g, int n, double x, int* i, double* w) {
  if (n == 1) {
    *i = 0;
    *w = 0.0;
    return;
  }
  int lo = 0;
  while (lo + 1 < n && g[lo + 1] <= x) ++lo;  // last grid point <= x (or 0 below the grid)
  if (lo > n - 2) lo = n - 2;
  *i = lo;
  *w = (x - g[lo]) / (g[lo + 1] - g[lo]);
}

double cost(const eagle_cost_table_t* t, double B, double L, double N) {
  int ib, il, in;
  double wb, wl, wn;
  axis_pos(t->B, t->nB, B, &ib, &wb);
  axis_pos(t->L, t->nL, L, &il, &wl);
  axis_pos(t->N, t->nN, N, &in, &wn);
  double total = 0.0;
  for (int db = 0; db < 2; ++db)
    for (int dl = 0; dl < 2; ++dl)
      for (int dn = 0; dn < 2; ++dn) {
        const double f = (db ? wb : 1.0 - wb) * (dl ? wl : 1.0 - wl) * (dn ? wn : 1.0 - wn);
        if (f != 0.0) total += f * t->us[((size_t)(ib + db) * t->nL + (il + dl)) * t->nN + (in + dn)];
      }
  return total;
}

}  // namespace

extern "C" {

EAGLE_API double eagle_cost_at(const eagle_cost_table_t* table, double B, double L, double N) {
  if (!valid_table(table) || !std::isfinite(B) || !std::isfinite(L) || !std::isfinite(N)) return NAN;
  return cost(table, B, L, N);
}

EAGLE_API eagle_status eagle_size_keep_level(const eagle_cost_table_t* table, double B, double L, int k, int level,
                                             const double* gains, int nb, double threshold, int* keep,
                                             double* ratio) {
  if (!table || !gains || !keep) return EAGLE_ERR_NULL;
  if (!valid_table(table)) return EAGLE_ERR_SHAPE;
  if (k <= 0 || level <= 0 || nb <= 0 || !std::isfinite(B) || !std::isfinite(L) || std::isnan(threshold))
    return EAGLE_ERR_SHAPE;
  const double dc = cost(table, B, L, (double)level * k) - cost(table, B, L, (double)(level - 1) * k);
  double g = 0.0;
  for (int b = 0; b < nb; ++b) g += gains[b];
  const double r = dc <= 0.0 ? INFINITY : g / dc;
  if (ratio) *ratio = r;
  *keep = r >= threshold ? 1 : 0;
  return EAGLE_OK;
}

EAGLE_API eagle_status eagle_size_level_width(const eagle_cost_table_t* table, double B, double L, int n_before,
                                             const double* logv, int k, int nb, double threshold, int* width,
                                             double* ratios) {
  if (!table || !logv || !width) return EAGLE_ERR_NULL;
  if (!valid_table(table)) return EAGLE_ERR_SHAPE;
  if (k <= 0 || nb <= 0 || n_before < 0 || !std::isfinite(B) || !std::isfinite(L) || std::isnan(threshold))
    return EAGLE_ERR_SHAPE;
  int w = 0;
  for (int j = 0; j < k; ++j) {
    double g = 0.0;
    for (int b = 0; b < nb; ++b) g += std::exp(logv[(size_t)b * k + j]);  // V = 0 for log V = -inf
    const double dc = cost(table, B, L, (double)(n_before + j + 1)) - cost(table, B, L, (double)(n_before + j));
    const double r = dc <= 0.0 ? INFINITY : g / dc;
    if (ratios) ratios[j] = r;
    if (!(g > 0.0 && r >= threshold)) {
      for (int i = j + 1; ratios && i < k; ++i) ratios[i] = NAN;  // not examined
      break;
    }
    w = j + 1;
  }
  *width = w;
  return EAGLE_OK;
}

}  // extern "C"

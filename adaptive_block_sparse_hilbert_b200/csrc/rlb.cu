// Runtime Load Balancing planner (host code).
//
// Method: aixai.ru FVAttn blog, section "Runtime Load Balancing (RLB)" -- after the mask
// is materialised, a few heavy heads are moved between ranks; a move is worth making when
// its net gain G = K - P - C is positive, K being the shortening of the critical path and
// P, C the communication and scheduling costs; each rank migrates at most one local head.
// PaperDaily article, 方法揭秘 -- per-rank loads, the heaviest head of the most loaded
// rank goes to the least loaded rank, repeated until the slowest / fastest ratio is below
// a threshold or the budget is used.
//
// On one GPU this plans for a virtual head split over n_ranks; it is host logic only.
#include <math.h>

#include <vector>

#include "fva_internal.cuh"

namespace {

// rank loads, each the sum of its heads' loads in head order
void loads_of(const double* load, const std::vector<int32_t>& rank_of, int n_ranks, std::vector<double>* out) {
  out->assign(n_ranks, 0.0);
  for (size_t h = 0; h < rank_of.size(); ++h) (*out)[rank_of[h]] += load[h];
}

int first_max(const std::vector<double>& L) {
  int r = 0;
  for (int i = 1; i < static_cast<int>(L.size()); ++i)
    if (L[i] > L[r]) r = i;
  return r;
}

int first_min(const std::vector<double>& L) {
  int r = 0;
  for (int i = 1; i < static_cast<int>(L.size()); ++i)
    if (L[i] < L[r]) r = i;
  return r;
}

}  // namespace

extern "C" FVA_API int fva_rlb_plan(const double* head_load_ms, int n_heads, int n_ranks, double comm_ms,
                                    double sched_ms, double threshold, int max_per_rank, int32_t* rank_of_out,
                                    fva_rlb_move* moves_out, int moves_capacity, int* n_moves_out) {
  if (!head_load_ms || !rank_of_out || !moves_out || !n_moves_out) return FVA_ERR_INVALID_ARG;
  if (n_heads < 1 || n_ranks < 1 || max_per_rank < 0 || !(threshold >= 1.0)) return FVA_ERR_INVALID_ARG;
  if (!(comm_ms >= 0.0) || !(sched_ms >= 0.0)) return FVA_ERR_INVALID_ARG;
  for (int h = 0; h < n_heads; ++h)
    if (!(head_load_ms[h] >= 0.0) || isinf(head_load_ms[h])) return FVA_ERR_INVALID_ARG;
  const int64_t budget = static_cast<int64_t>(n_ranks) * max_per_rank;
  if (moves_capacity < (budget < n_heads ? budget : n_heads)) return FVA_ERR_CAPACITY;

  std::vector<int32_t> home(n_heads), rank_of(n_heads);
  for (int r = 0; r < n_ranks; ++r) {
    const int lo = static_cast<int>(static_cast<int64_t>(r) * n_heads / n_ranks);
    const int hi = static_cast<int>(static_cast<int64_t>(r + 1) * n_heads / n_ranks);
    for (int h = lo; h < hi; ++h) home[h] = rank_of[h] = r;
  }
  std::vector<int> exported(n_ranks, 0);
  std::vector<double> L, L_try;
  int n = 0;
  while (true) {
    loads_of(head_load_ms, rank_of, n_ranks, &L);
    const int r_max = first_max(L), r_min = first_min(L);
    const double mx = L[r_max], mn = L[r_min];
    if (mn > 0.0 && mx / mn < threshold) break;  // balanced enough (an idle rank never is)
    if (r_max == r_min || exported[r_max] >= max_per_rank) break;
    // the most loaded rank's own heads, heaviest first; the first whose move pays is taken
    std::vector<int> own;
    for (int h = 0; h < n_heads; ++h)
      if (rank_of[h] == r_max && home[h] == r_max) own.push_back(h);
    for (size_t i = 1; i < own.size(); ++i) {  // insertion sort: load desc, index asc
      const int h = own[i];
      size_t j = i;
      while (j > 0 && (head_load_ms[own[j - 1]] < head_load_ms[h] ||
                       (head_load_ms[own[j - 1]] == head_load_ms[h] && own[j - 1] > h))) {
        own[j] = own[j - 1];
        --j;
      }
      own[j] = h;
    }
    int chosen = -1;
    double gain = 0.0;
    for (int h : own) {
      rank_of[h] = r_min;
      loads_of(head_load_ms, rank_of, n_ranks, &L_try);
      rank_of[h] = r_max;
      const double g = (mx - L_try[first_max(L_try)]) - comm_ms - sched_ms;
      if (g > 0.0) {
        chosen = h;
        gain = g;
        break;
      }
    }
    if (chosen < 0) break;
    rank_of[chosen] = r_min;
    ++exported[r_max];
    moves_out[n].head = chosen;
    moves_out[n].from_rank = r_max;
    moves_out[n].to_rank = r_min;
    moves_out[n].reserved = 0;
    moves_out[n].gain_ms = gain;
    ++n;
  }
  for (int h = 0; h < n_heads; ++h) rank_of_out[h] = rank_of[h];
  *n_moves_out = n;
  return FVA_OK;
}

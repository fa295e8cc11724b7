// Host balance planner over the dispatch layout's per-expert counts.
//
// Sources: the DeepEP pull request "Intra-node compute compensation + overlap
// robustness (CUDA719 fix)", Python section (a water-filling chunk-migration
// planner with expert-affinity batching, a makespan guard, a cost-aware no-op
// and a 128-aligned fine-balance pass), and the TEMPO summary, section 2
// (max-affine expert time t = max(a + b*G, c + beta*N), G activated expert
// replicas and N tokens on a GPU; the tile-aware form adds b2 * (tiles - G),
// a tile being a 128-token M-tile of section 1).
//
// Logical rank r starts with the contiguous experts [r*E/R, (r+1)*E/R).  A
// step pairs the most expensive rank (src) with the cheapest (dst) and moves
// 128-token chunks of one expert between them: experts already present on
// dst are tried first (no new replica), then those with the most tokens on
// src.  The water-filling pass moves as many whole chunks as keep dst no more
// expensive than src; the fine pass moves one chunk.  A move is kept only if
// it lowers the makespan by more than min_gain.  Costs are doubles evaluated
// term by term in a fixed order (this file is compiled without contraction),
// so the plan is reproducible bit for bit.
#include <stdint.h>

#include <algorithm>
#include <vector>

#include "moe_dispatch.h"

namespace {

constexpr int64_t kChunk = MOE_TILE_M;

struct Planner {
  int E, R;
  moe_cost_model_t cost;
  std::vector<int64_t> tok;   // [R][E] tokens of expert e processed on rank r
  std::vector<int64_t> mig;   // [R] tokens migrated into rank r

  int64_t& at(int r, int e) { return tok[(size_t)r * E + e]; }

  double rank_cost_of(const int64_t* row, int64_t migrated_in) const {
    int64_t G = 0, N = 0, tiles = 0;
    for (int e = 0; e < E; ++e) {
      const int64_t n = row[e];
      if (n > 0) {
        G += 1;
        N += n;
        tiles += (n + kChunk - 1) / kChunk;
      }
    }
    const double t1 = cost.a + cost.b * (double)G + cost.b2 * (double)(tiles - G);
    const double t2 = cost.c + cost.beta * (double)N;
    return (t1 > t2 ? t1 : t2) + cost.mig * (double)migrated_in;
  }
  double rank_cost(int r) const { return rank_cost_of(&tok[(size_t)r * E], mig[r]); }

  double makespan() const {
    double m = rank_cost(0);
    for (int r = 1; r < R; ++r) {
      const double c = rank_cost(r);
      if (c > m) m = c;
    }
    return m;
  }

  // costs of src and dst after moving n tokens of e
  void trial(int src, int dst, int e, int64_t n, double* ts, double* td) {
    at(src, e) -= n;
    at(dst, e) += n;
    *ts = rank_cost_of(&tok[(size_t)src * E], mig[src]);
    *td = rank_cost_of(&tok[(size_t)dst * E], mig[dst] + n);
    at(src, e) += n;
    at(dst, e) -= n;
  }

  int64_t chunk_for(int src, int dst, int e, bool fine) {
    const int64_t have = at(src, e);
    const int64_t one = have > kChunk ? kChunk : have;
    if (fine) return one;
    for (int64_t k = (have + kChunk - 1) / kChunk; k >= 1; --k) {
      const int64_t n = k * kChunk < have ? k * kChunk : have;
      double ts, td;
      trial(src, dst, e, n, &ts, &td);
      if (td <= ts) return n;
    }
    return one;
  }
};

}  // namespace

extern "C" int moe_plan_balance(const int32_t* expert_counts, int E, int R,
                                const moe_cost_model_t* cost, double min_gain, int max_moves,
                                moe_move_t* moves, int* n_moves, double* makespan_before,
                                double* makespan_after) {
  if (!expert_counts || !cost || !n_moves || E < 1 || E > MOE_MAX_EXPERTS || R < 1 || R > E ||
      E % R != 0 || max_moves < 0 || (max_moves > 0 && !moves) || !(min_gain >= 0.0))
    return MOE_ERR_INVALID_ARG;
  for (int e = 0; e < E; ++e)
    if (expert_counts[e] < 0) return MOE_ERR_INVALID_ARG;

  Planner p;
  p.E = E;
  p.R = R;
  p.cost = *cost;
  p.tok.assign((size_t)R * E, 0);
  p.mig.assign((size_t)R, 0);
  const int El = E / R;
  for (int e = 0; e < E; ++e) p.at(e / El, e) = expert_counts[e];

  const double before = p.makespan();
  int made = 0;
  std::vector<int> cands;
  std::vector<double> costs((size_t)R);
  for (int pass = 0; pass < 2; ++pass) {
    const bool fine = pass == 1;
    while (made < max_moves) {
      for (int r = 0; r < R; ++r) costs[r] = p.rank_cost(r);
      int src = 0, dst = 0;
      for (int r = 1; r < R; ++r) {
        if (costs[r] > costs[src]) src = r;
        if (costs[r] < costs[dst]) dst = r;
      }
      if (src == dst) break;
      cands.clear();
      for (int e = 0; e < E; ++e)
        if (p.at(src, e) > 0) cands.push_back(e);
      std::sort(cands.begin(), cands.end(), [&](int x, int y) {
        const int px = p.at(dst, x) > 0 ? 0 : 1, py = p.at(dst, y) > 0 ? 0 : 1;
        if (px != py) return px < py;
        if (p.at(src, x) != p.at(src, y)) return p.at(src, x) > p.at(src, y);
        return x < y;
      });
      bool kept = false;
      for (int e : cands) {
        const int64_t n = p.chunk_for(src, dst, e, fine);
        p.at(src, e) -= n;
        p.at(dst, e) += n;
        p.mig[dst] += n;
        if (p.makespan() < costs[src] - min_gain) {
          moves[made].expert = e;
          moves[made].src_rank = src;
          moves[made].dst_rank = dst;
          moves[made].tokens = (int32_t)n;
          ++made;
          kept = true;
          break;
        }
        p.at(src, e) += n;
        p.at(dst, e) -= n;
        p.mig[dst] -= n;
      }
      if (!kept) break;
    }
  }
  *n_moves = made;
  if (makespan_before) *makespan_before = before;
  if (makespan_after) *makespan_after = p.makespan();
  return MOE_OK;
}

// Host-side planning of the order of the pairs inside each stage.
//
// The pairs of a stage are disjoint (page "ParoQuant: pairwise rotations that
// survive deployment", section "A rotation small enough to execute"), so they
// may be applied in any order, and a pair (i, j) with (cos, sin) is the same
// rotation as (j, i) with (cos, -sin).  The transform kernels give pair t of a
// stage to lane t % 32 of a warp and load channel i, then channel j, of every
// pair from a shared-memory plane where channel c sits in bank c % 32.  This
// planner reorders (and where needed flips) the pairs of every stage so that
// every aligned group of 32 consecutive pairs has 32 distinct i % 32 and 32
// distinct j % 32: each of those loads and stores is then one conflict-free
// shared-memory wavefront.
//
// Construction, per stage: take the multigraph on the 32 residues with one edge
// (i % 32, j % 32) per pair.  Every channel appears once per stage, so every
// residue has degree d / 32; when that is even (d % 64 == 0) an Euler circuit of
// each component orients the edges so that every residue is the i-side of d/64
// pairs and the j-side of d/64 pairs.  The resulting bipartite multigraph
// (i-residue -> j-residue) is d/64-regular and splits into d/64 perfect
// matchings (Hall / Konig); each matching is one group of 32 pairs.
//
// Kernels that keep several rows of a channel side by side (a float2 or float4
// per channel) access shared memory in phases of 16 or 8 lanes, so each group
// of 32 is then ordered so that every aligned 16 has distinct i % 16 and
// j % 16, and every aligned 8 distinct i % 8 and j % 8: n pairs with distinct
// residues mod n hold every residue mod n/2 twice on each side, a 2-regular
// bipartite multigraph, which splits into two perfect matchings.
#include <cstring>
#include <functional>
#include <vector>

#include "paro_internal.cuh"

namespace {

constexpr int kBanks = 32;

struct Edge {
  int u, v;      // residues as stored (i % 32, j % 32)
  int pair;      // index of the pair in the stage
  bool flip;     // traversed v -> u by the Euler circuit
  bool used;
};

// Euler circuits of every component; orients each edge along the walk.
void orient(std::vector<Edge>& E, int nodes) {
  std::vector<std::vector<int>> adj(nodes);
  for (int e = 0; e < (int)E.size(); ++e) {
    adj[E[e].u].push_back(e);
    if (E[e].v != E[e].u) adj[E[e].v].push_back(e);
  }
  std::vector<size_t> next(nodes, 0);
  std::vector<bool> done(E.size(), false);
  for (int start = 0; start < nodes; ++start) {
    // Hierholzer, iterative; the orientation of an edge is the direction it is
    // first walked in, which yields in-degree == out-degree at every node
    std::vector<int> stack{start};
    while (!stack.empty()) {
      const int x = stack.back();
      while (next[x] < adj[x].size() && done[adj[x][next[x]]]) ++next[x];
      if (next[x] == adj[x].size()) {
        stack.pop_back();
        continue;
      }
      const int e = adj[x][next[x]];
      done[e] = true;
      const int y = (E[e].u == x) ? E[e].v : E[e].u;
      E[e].flip = (E[e].u != x);  // walked v -> u
      stack.push_back(y);
    }
  }
}

// One perfect matching of the remaining edges (left = i-residue, right = j-residue).
bool perfect_matching(const std::vector<Edge>& E, const std::vector<std::vector<int>>& out_edges,
                      std::vector<int>& match_edge_of_left) {
  std::vector<int> left_of_right(kBanks, -1), edge_of_left(kBanks, -1);
  auto right = [&](const Edge& e) { return e.flip ? e.u : e.v; };
  for (int l = 0; l < kBanks; ++l) {
    std::vector<bool> seen(kBanks, false);
    // augmenting path search (Kuhn's algorithm), depth at most 32
    std::function<bool(int)> try_left = [&](int x) -> bool {
      for (int e : out_edges[x]) {
        if (E[e].used) continue;
        const int r = right(E[e]);
        if (seen[r]) continue;
        seen[r] = true;
        if (left_of_right[r] < 0 || try_left(left_of_right[r])) {
          left_of_right[r] = x;
          edge_of_left[x] = e;
          return true;
        }
      }
      return false;
    };
    if (!try_left(l)) return false;
  }
  match_edge_of_left = edge_of_left;
  return true;
}

// Orders the 2n pairs of `grp` (oriented i -> j, distinct i % 2n and j % 2n)
// into two halves of n with distinct residues mod n, recursively down to 8.
void split_phases(std::vector<std::pair<int, int>>& grp) {
  const int n2 = (int)grp.size(), n = n2 / 2;
  if (n < 8) return;
  std::vector<int> left_of_right(n, -1), edge_of_left(n, -1);
  std::vector<std::vector<int>> out(n);
  for (int e = 0; e < n2; ++e) out[grp[e].first % n].push_back(e);
  for (int l = 0; l < n; ++l) {
    std::vector<bool> seen(n, false);
    std::function<bool(int)> try_left = [&](int x) -> bool {
      for (int e : out[x]) {
        const int r = grp[e].second % n;
        if (seen[r]) continue;
        seen[r] = true;
        if (left_of_right[r] < 0 || try_left(left_of_right[r])) {
          left_of_right[r] = x;
          edge_of_left[x] = e;
          return true;
        }
      }
      return false;
    };
    try_left(l);  // a 2-regular bipartite multigraph always has a perfect matching
  }
  std::vector<bool> first(n2, false);
  for (int l = 0; l < n; ++l)
    if (edge_of_left[l] >= 0) first[edge_of_left[l]] = true;
  std::vector<std::pair<int, int>> a, b;
  for (int e = 0; e < n2; ++e) (first[e] ? a : b).push_back(grp[e]);
  if ((int)a.size() != n) return;  // cannot happen; keep the mod-2n order
  split_phases(a);
  split_phases(b);
  for (int e = 0; e < n; ++e) {
    grp[e] = a[e];
    grp[n + e] = b[e];
  }
}

}  // namespace

extern "C" paro_status paro_plan_pair_order(const uint16_t* h_pairs, const float* h_cos, const float* h_sin, int K,
                                            int d, uint16_t* h_pairs_out, float* h_cos_out, float* h_sin_out) {
  if (K < 0 || K > paro::kMaxStages) return paro::record_error(PARO_ERR_INVALID_ARG, "K = %d out of range", K);
  if (d < 2 || (d & 1)) return paro::record_error(PARO_ERR_INVALID_ARG, "d = %d must be even", d);
  if (K > 0 && (!h_pairs || !h_cos || !h_sin || !h_pairs_out || !h_cos_out || !h_sin_out))
    return paro::record_error(PARO_ERR_INVALID_ARG, "null table pointer");
  if (d % (2 * kBanks))
    return paro::record_error(PARO_ERR_UNSUPPORTED, "d = %d is not a multiple of 64: no conflict-free order planned", d);
  const int half = d / 2, D = d / (2 * kBanks);
  for (int k = 0; k < K; ++k) {
    const uint16_t* P = h_pairs + (size_t)k * half * 2;
    // the stage must be a perfect matching of 0..d-1
    std::vector<char> seen(d, 0);
    for (int t = 0; t < 2 * half; ++t) {
      const int c = P[t];
      if (c >= d || seen[c])
        return paro::record_error(PARO_ERR_INVALID_ARG, "stage %d is not a perfect matching of the %d channels", k, d);
      seen[c] = 1;
    }
    std::vector<Edge> E(half);
    for (int t = 0; t < half; ++t) E[t] = Edge{P[2 * t] % kBanks, P[2 * t + 1] % kBanks, t, false, false};
    orient(E, kBanks);
    std::vector<std::vector<int>> out_edges(kBanks);
    for (int e = 0; e < half; ++e) out_edges[E[e].flip ? E[e].v : E[e].u].push_back(e);
    for (int g = 0; g < D; ++g) {
      std::vector<int> m;
      if (!perfect_matching(E, out_edges, m))
        return paro::record_error(PARO_ERR_CUDA, "internal: stage %d has no perfect matching left", k);
      // the group's pairs, oriented (i, j)
      std::vector<std::pair<int, int>> grp(kBanks);
      std::vector<int> edge_at(kBanks);
      for (int l = 0; l < kBanks; ++l) {
        const Edge& e = E[m[l]];
        const int t = e.pair;
        const int i = e.flip ? P[2 * t + 1] : P[2 * t], j = e.flip ? P[2 * t] : P[2 * t + 1];
        grp[l] = {i, j};
      }
      split_phases(grp);
      // map each ordered (i, j) back to its edge: i determines the edge within the group
      for (int l = 0; l < kBanks; ++l) {
        int found = -1;
        for (int q = 0; q < kBanks; ++q) {
          const Edge& e = E[m[q]];
          const int t = e.pair;
          const int i = e.flip ? P[2 * t + 1] : P[2 * t];
          if (i == grp[l].first) { found = m[q]; break; }
        }
        edge_at[l] = found;
      }
      for (int l = 0; l < kBanks; ++l) {
        Edge& e = E[edge_at[l]];
        e.used = true;
        const int t = e.pair, o = g * kBanks + l;
        const uint16_t i = P[2 * t], j = P[2 * t + 1];
        h_pairs_out[(size_t)k * half * 2 + 2 * o] = e.flip ? j : i;
        h_pairs_out[(size_t)k * half * 2 + 2 * o + 1] = e.flip ? i : j;
        h_cos_out[(size_t)k * half + o] = h_cos[(size_t)k * half + t];
        h_sin_out[(size_t)k * half + o] = e.flip ? -h_sin[(size_t)k * half + t] : h_sin[(size_t)k * half + t];
      }
    }
  }
  return PARO_OK;
}

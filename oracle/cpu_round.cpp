// Test and measurement infrastructure: the oracle's greedy (T = 0) round
// restated in plain C++ (fp64), run on all host cores with OpenMP.  It is the
// multi-core CPU baseline that bench.py times next to the numpy oracle, and it
// is checked against that oracle by tests/test_oracle_cpu_round.py.  Nothing
// in the library links it.
//
// Steps, in the order of the numpy oracle (oracle/markov_tree.py,
// oracle/verify_attn.py, oracle/accept.py):
//  * build: sequential best-first over a max-heap ordered by (fp32 key desc,
//    depth asc, parent index asc, rank asc); expanding a node at depth d with
//    token t computes z[x] = L[d][x] + sum_rho A[t][rho] Bt[x][rho] over the
//    vocabulary, s = z (T = 0), lse = log sum exp s, and its k best tokens
//    (ties to the lower id); child j of a node gets key(parent) + (s_(j) - lse)
//    (identity calibration, lambda = 0) (PCTree summary, DSpark and "k=4, N=32"
//    paragraphs; TreeSpark article, "core idea");
//  * verify: per (row, head) softmax(scale q.k) v over the prefix, the root
//    and the row's ancestors (TreeSpark article, introduction);
//  * accept: follow the child equal to each row's target argmax (ties to the
//    lower id); the bonus is the argmax at the stop node (PCTree summary,
//    setup: greedy verification).
#include <omp.h>
#include <stdint.h>

#include <algorithm>
#include <cmath>
#include <queue>
#include <utility>
#include <vector>

namespace {

struct Item {
  float negk;   // -fp32(key)
  int depth, parent, rank;
  double key;
  int token;
  bool operator>(const Item& o) const {  // min-heap on (negk, depth, parent, rank)
    if (negk != o.negk) return negk > o.negk;
    if (depth != o.depth) return depth > o.depth;
    if (parent != o.parent) return parent > o.parent;
    return rank > o.rank;
  }
};

// z, lse and the k best tokens of one node's distribution
void expand(const float* L, const float* A, const float* Bt, int V, int r, int k, int depth,
            int token, std::vector<int>& kids, std::vector<double>& logq) {
  std::vector<double> z(V);
  const float* a = A + (size_t)token * r;
  const float* l = L + (size_t)depth * V;
#pragma omp parallel for schedule(static)
  for (int x = 0; x < V; ++x) {
    const float* b = Bt + (size_t)x * r;
    double acc = 0.0;
    for (int p = 0; p < r; ++p) acc += (double)a[p] * (double)b[p];
    z[x] = (double)l[x] + acc;
  }
  double mx = -INFINITY;
#pragma omp parallel for reduction(max : mx)
  for (int x = 0; x < V; ++x) mx = std::max(mx, z[x]);
  double se = 0.0;
#pragma omp parallel for reduction(+ : se)
  for (int x = 0; x < V; ++x) se += std::exp(z[x] - mx);
  const double lse = mx + std::log(se);
  // k best: every thread its own list, then one merge (ties to the lower id)
  auto better = [&](int x, int y) { return z[x] > z[y] || (z[x] == z[y] && x < y); };
  const int nt = omp_get_max_threads();
  std::vector<std::vector<int>> part(nt);
#pragma omp parallel
  {
    std::vector<int>& mine = part[omp_get_thread_num()];
#pragma omp for schedule(static)
    for (int x = 0; x < V; ++x) {
      if ((int)mine.size() < k) {
        mine.push_back(x);
        std::sort(mine.begin(), mine.end(), better);
      } else if (better(x, mine.back())) {
        mine.back() = x;
        std::sort(mine.begin(), mine.end(), better);
      }
    }
  }
  std::vector<int> all;
  for (auto& p : part) all.insert(all.end(), p.begin(), p.end());
  std::sort(all.begin(), all.end(), better);
  kids.assign(all.begin(), all.begin() + std::min<size_t>(k, all.size()));
  logq.resize(kids.size());
  for (size_t j = 0; j < kids.size(); ++j) logq[j] = z[kids[j]] - lse;
}

}  // namespace

extern "C" int cpu_round_t0(const float* L, const float* A, const float* Bt, int V, int r, int Bk,
                            int k, int N, int root, const float* q, const float* kp,
                            const float* vp, const float* kt, const float* vt, int P, int Hq,
                            int Hkv, int d, double scale, const float* target, int32_t* tokens,
                            int32_t* parents, int32_t* depths, double* keys, int32_t* n_nodes,
                            double* attn_out, int32_t* acc_nodes, int32_t* n_acc,
                            int32_t* bonus) {
  if (V < 1 || r < 1 || Bk < 1 || k < 1 || k > V || N < 0 || N > 64 || root < 0 || root >= V)
    return 1;
  // ---- build
  std::priority_queue<Item, std::vector<Item>, std::greater<Item>> heap;
  std::vector<int> kids;
  std::vector<double> logq;
  auto push = [&](int depth, int token, int parent, double pkey) {
    expand(L, A, Bt, V, r, k, depth, token, kids, logq);
    for (size_t j = 0; j < kids.size(); ++j) {
      const double key = pkey + std::min(0.0, logq[j]);
      heap.push(Item{-(float)key, depth + 1, parent, (int)j, key, kids[j]});
    }
  };
  if (N > 0) push(0, root, -1, 0.0);
  std::vector<uint64_t> anc;
  int n = 0;
  while (n < N && !heap.empty()) {
    const Item it = heap.top();
    heap.pop();
    tokens[n] = it.token;
    parents[n] = it.parent;
    depths[n] = it.depth;
    keys[n] = it.key;
    anc.push_back((it.parent < 0 ? 0ull : anc[it.parent]) | (1ull << n));
    ++n;
    if (it.depth < Bk) push(it.depth, it.token, n - 1, it.key);
  }
  *n_nodes = n;
  // ---- verify: rows 0 (root) .. n
  const int g = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int i = 0; i <= n; ++i)
    for (int h = 0; h < Hq; ++h) {
      const int kv = h / g;
      std::vector<int> cols;  // tree columns: 0 = root, j + 1 = node j
      cols.push_back(0);
      if (i >= 1)
        for (int j = 0; j < n; ++j)
          if ((anc[i - 1] >> j) & 1ull) cols.push_back(j + 1);
      const float* qi = q + ((size_t)i * Hq + h) * d;
      std::vector<double> sc(P + cols.size());
      double mx = -INFINITY;
      for (int j = 0; j < P; ++j) {
        const float* kj = kp + ((size_t)j * Hkv + kv) * d;
        double s = 0.0;
        for (int e = 0; e < d; ++e) s += (double)qi[e] * kj[e];
        sc[j] = scale * s;
        mx = std::max(mx, sc[j]);
      }
      for (size_t c = 0; c < cols.size(); ++c) {
        const float* kj = kt + ((size_t)cols[c] * Hkv + kv) * d;
        double s = 0.0;
        for (int e = 0; e < d; ++e) s += (double)qi[e] * kj[e];
        sc[P + c] = scale * s;
        mx = std::max(mx, sc[P + c]);
      }
      double den = 0.0;
      for (double& s : sc) den += (s = std::exp(s - mx));
      double* o = attn_out + ((size_t)i * Hq + h) * d;
      for (int e = 0; e < d; ++e) o[e] = 0.0;
      for (int j = 0; j < P; ++j) {
        const float* vj = vp + ((size_t)j * Hkv + kv) * d;
        for (int e = 0; e < d; ++e) o[e] += sc[j] * vj[e];
      }
      for (size_t c = 0; c < cols.size(); ++c) {
        const float* vj = vt + ((size_t)cols[c] * Hkv + kv) * d;
        for (int e = 0; e < d; ++e) o[e] += sc[P + c] * vj[e];
      }
      for (int e = 0; e < d; ++e) o[e] /= den;
    }
  // ---- accept: every row's argmax, then the walk
  std::vector<int> am(n + 1);
#pragma omp parallel for
  for (int i = 0; i <= n; ++i) {
    const float* t = target + (size_t)i * V;
    int best = 0;
    for (int x = 1; x < V; ++x)
      if (t[x] > t[best]) best = x;
    am[i] = best;
  }
  int node = -1, na = 0, a = 0;
  while (true) {
    a = am[node + 1];
    int next = -1;
    for (int i = 0; i < n && next < 0; ++i)
      if (parents[i] == node && tokens[i] == a) next = i;
    if (next < 0 || na >= Bk) break;
    acc_nodes[na++] = next;
    node = next;
  }
  *n_acc = na;
  *bonus = a;
  return 0;
}

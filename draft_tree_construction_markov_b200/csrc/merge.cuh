// Warp-level merges of the per-CTA partial results that the node-batched GEMM
// writes for every node row: (max, sum exp) pairs into a log-sum-exp, and
// sorted top-k lists into the row's best entries (ties to the lower token).
// Layout per node row: statistics [ncta], list entries [k][ncta] (entry i of
// every CTA contiguous).
#pragma once
#include "build.cuh"

namespace dt {

// (v1, i1) ranks before (v2, i2): larger value first, then lower token.
__device__ __forceinline__ bool ranks_first(float v1, int32_t i1, float v2, int32_t i2) {
  return v1 > v2 || (v1 == v2 && i1 < i2);
}

// Insert (v, id) into a register list sorted by ranks_first; the caller
// guarantees that it ranks before the k-th entry.  Entries past k are scratch.
template <int KMAX>
__device__ __forceinline__ void list_insert(float (&L)[KMAX], int32_t (&I)[KMAX], float v,
                                            int32_t id) {
  float nl[KMAX];
  int32_t ni[KMAX];
#pragma unroll
  for (int i = 0; i < KMAX; ++i) {
    const bool keep = ranks_first(L[i], I[i], v, id);
    const bool keep_prev = i > 0 && ranks_first(L[i - 1], I[i - 1], v, id);
    nl[i] = keep ? L[i] : ((i == 0 || keep_prev) ? v : L[i - 1]);
    ni[i] = keep ? I[i] : ((i == 0 || keep_prev) ? id : I[i - 1]);
  }
#pragma unroll
  for (int i = 0; i < KMAX; ++i) {
    L[i] = nl[i];
    I[i] = ni[i];
  }
}

template <int KMAX>
__device__ __forceinline__ void list_entry(const float (&L)[KMAX], const int32_t (&I)[KMAX], int j,
                                           float& v, int32_t& id) {
  v = L[0];
  id = I[0];
#pragma unroll
  for (int i = 1; i < KMAX; ++i)
    if (i == j) {
      v = L[i];
      id = I[i];
    }
}

// Fold JP loaded partial lists (each sorted, k long) into the lane's private
// list of the kb best.  Entry bar: the best kb-th entry of any partial (its
// partial alone holds kb entries at or above it), so lower entries are skipped.
template <int KMAX, int JP>
__device__ __forceinline__ void fold_lists(const float (&pv)[JP][KMAX], const int32_t (&pi)[JP][KMAX],
                                           int kb, float (&L)[KMAX], int32_t (&I)[KMAX]) {
  float bv = -INFINITY;
  int32_t bi = 0x7fffffff;
#pragma unroll
  for (int j = 0; j < JP; ++j) {
    float v;
    int32_t id;
    list_entry<KMAX>(pv[j], pi[j], kb - 1, v, id);
    if (ranks_first(v, id, bv, bi)) {
      bv = v;
      bi = id;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int32_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ranks_first(ov, oi, bv, bi)) {
      bv = ov;
      bi = oi;
    }
  }
#pragma unroll
  for (int j = 0; j < JP; ++j) {
#pragma unroll
    for (int i = 0; i < KMAX; ++i) {
      if (ranks_first(bv, bi, pv[j][i], pi[j][i])) break;  // lists are sorted
      float kv;
      int32_t ki;
      list_entry<KMAX>(L, I, kb - 1, kv, ki);
      if (ranks_first(pv[j][i], pi[j][i], kv, ki)) list_insert<KMAX>(L, I, pv[j][i], pi[j][i]);
    }
  }
}

// kb rounds of a warp-wide arg-best over the lanes' private lists; lane 0
// writes the winners.  out_v / out_i may be NULL.
template <int KMAX>
__device__ __forceinline__ void emit_best(float (&L)[KMAX], int32_t (&I)[KMAX], int kb, int lane,
                                          float* out_v, int32_t* out_i) {
  for (int j = 0; j < kb; ++j) {
    float wv = L[0];
    int32_t wi = I[0];
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, wv, o);
      const int32_t oi = __shfl_xor_sync(0xffffffffu, wi, o);
      if (ranks_first(ov, oi, wv, wi)) {
        wv = ov;
        wi = oi;
      }
    }
    if (L[0] == wv && I[0] == wi) {  // (value, token) pairs are unique: one owner
#pragma unroll
      for (int i = 0; i + 1 < KMAX; ++i) {
        L[i] = L[i + 1];
        I[i] = I[i + 1];
      }
      L[KMAX - 1] = -INFINITY;
      I[KMAX - 1] = 0x7fffffff;
    }
    if (lane == 0) {
      if (out_v) out_v[j] = wv;
      if (out_i) out_i[j] = wi;
    }
  }
}

template <int KMAX>
__device__ __forceinline__ void list_init(float (&L)[KMAX], int32_t (&I)[KMAX]) {
#pragma unroll
  for (int i = 0; i < KMAX; ++i) {
    L[i] = -INFINITY;
    I[i] = 0x7fffffff;
  }
}

__device__ __forceinline__ void lse_fold(float2 p, float& m, float& sv) {
  constexpr float kL2e = 1.4426950408889634f;
  if (p.x == -INFINITY) return;
  if (p.x > m) {
    sv = sv * exp2f((m - p.x) * kL2e) + p.y;
    m = p.x;
  } else {
    sv += p.y * exp2f((p.x - m) * kL2e);
  }
}

__device__ __forceinline__ float lse_finish(float m, float sv) {
  constexpr float kL2e = 1.4426950408889634f;
  const float wm = warp_max(m);
  float ws = (m == -INFINITY) ? 0.f : sv * exp2f((m - wm) * kL2e);
  ws = warp_sum(ws);
  return wm + logf(ws);
}

// The kb best entries of JP loaded partial lists per lane, written by lane 0.
// Usually only a handful of entries can reach the kb best: those at or above
// the entry bar (the best kb-th entry of any partial), and only the first kb
// of each sorted list.  They are compacted into the warp's scratch (32 slots)
// and chosen with kb rounds of a warp arg-best over one entry per lane.  When
// more than 32 qualify (heavy ties), the lists are folded instead.
template <int KMAX, int JP>
__device__ __forceinline__ void select_best(const float (&pv)[JP][KMAX],
                                            const int32_t (&pi)[JP][KMAX], int kb, int lane,
                                            float* sv, int32_t* si, float* out_v,
                                            int32_t* out_i) {
  float bv = -INFINITY;
  int32_t bi = 0x7fffffff;
#pragma unroll
  for (int j = 0; j < JP; ++j) {
    float v;
    int32_t id;
    list_entry<KMAX>(pv[j], pi[j], kb - 1, v, id);
    if (ranks_first(v, id, bv, bi)) {
      bv = v;
      bi = id;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int32_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ranks_first(ov, oi, bv, bi)) {
      bv = ov;
      bi = oi;
    }
  }
  int cnt = 0;
#pragma unroll
  for (int j = 0; j < JP; ++j)
#pragma unroll
    for (int i = 0; i < KMAX; ++i)
      cnt += (i < kb && !ranks_first(bv, bi, pv[j][i], pi[j][i])) ? 1 : 0;
  const int total = __reduce_add_sync(0xffffffffu, cnt);
  if (total > 32) {
    float L[KMAX];
    int32_t I[KMAX];
    list_init<KMAX>(L, I);
    fold_lists<KMAX, JP>(pv, pi, kb, L, I);
    emit_best<KMAX>(L, I, kb, lane, out_v, out_i);
    return;
  }
  int base = 0;
  const unsigned below = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < JP; ++j)
#pragma unroll
    for (int i = 0; i < KMAX; ++i) {
      const bool q = i < kb && !ranks_first(bv, bi, pv[j][i], pi[j][i]);
      const unsigned m = __ballot_sync(0xffffffffu, q);
      if (q) {
        const int slot = base + __popc(m & below);
        sv[slot] = pv[j][i];
        si[slot] = pi[j][i];
      }
      base += __popc(m);
    }
  __syncwarp();
  float v = lane < total ? sv[lane] : -INFINITY;
  int32_t id = lane < total ? si[lane] : 0x7fffffff;
  __syncwarp();
  for (int r = 0; r < kb; ++r) {
    float wv = v;
    int32_t wi = id;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, wv, o);
      const int32_t oi = __shfl_xor_sync(0xffffffffu, wi, o);
      if (ranks_first(ov, oi, wv, wi)) {
        wv = ov;
        wi = oi;
      }
    }
    if (v == wv && id == wi) {  // unique (value, token): one owner
      v = -INFINITY;
      id = 0x7fffffff;
    }
    if (lane == 0) {
      if (out_v) out_v[r] = wv;
      if (out_i) out_i[r] = wi;
    }
  }
}

// One warp merges everything the frontier needs of one node's ncta partials:
// its log-sum-exp, the kb best values of s (and their tokens when out_i is
// given) and, when GV is given, the tokens of the kb best Gumbel keys.  Each
// lane issues the loads of all its partials (statistics and lists) before it
// uses any of them, so one memory round trip serves the whole merge.
template <int KMAX>
__device__ __forceinline__ float merge_node(const float2* PS, const float* PV, const int32_t* PI,
                                            const float* GV, const int32_t* GI, int ncta, int k,
                                            int kb, int lane, float* out_v, int32_t* out_i,
                                            int32_t* out_g, float* sv, int32_t* si) {
  constexpr int JP = KMAX <= 4 ? 5 : 1;
  float m = -INFINITY, sum = 0.f;
  if (ncta <= 32 * JP) {
    // every partial in one load batch; compacted selection
    float2 ps[JP];
    float pv[JP][KMAX], gv[JP][KMAX];
    int32_t pi[JP][KMAX], gi[JP][KMAX];
#pragma unroll
    for (int j = 0; j < JP; ++j) {
      const int c = 32 * j + lane;
      ps[j] = c < ncta ? __ldcg(PS + c) : make_float2(-INFINITY, 0.f);
#pragma unroll
      for (int i = 0; i < KMAX; ++i) {
        const bool in = c < ncta && i < k;
        pv[j][i] = in ? __ldcg(PV + (size_t)i * ncta + c) : -INFINITY;
        pi[j][i] = in ? __ldcg(PI + (size_t)i * ncta + c) : 0x7fffffff;
        gv[j][i] = (in && GV) ? __ldcg(GV + (size_t)i * ncta + c) : -INFINITY;
        gi[j][i] = (in && GV) ? __ldcg(GI + (size_t)i * ncta + c) : 0x7fffffff;
      }
    }
#pragma unroll
    for (int j = 0; j < JP; ++j) lse_fold(ps[j], m, sum);
    select_best<KMAX, JP>(pv, pi, kb, lane, sv, si, out_v, out_i);
    if (GV) select_best<KMAX, JP>(gv, gi, kb, lane, sv, si, nullptr, out_g);
    return lse_finish(m, sum);
  }
  float L[KMAX], G[KMAX];
  int32_t I[KMAX], GI_[KMAX];
  list_init<KMAX>(L, I);
  list_init<KMAX>(G, GI_);
  for (int c0 = 0; c0 < ncta; c0 += 32 * JP) {
    float2 ps[JP];
    float pv[JP][KMAX], gv[JP][KMAX];
    int32_t pi[JP][KMAX], gi[JP][KMAX];
#pragma unroll
    for (int j = 0; j < JP; ++j) {
      const int c = c0 + 32 * j + lane;
      ps[j] = c < ncta ? __ldcg(PS + c) : make_float2(-INFINITY, 0.f);
#pragma unroll
      for (int i = 0; i < KMAX; ++i) {
        const bool in = c < ncta && i < k;
        pv[j][i] = in ? __ldcg(PV + (size_t)i * ncta + c) : -INFINITY;
        pi[j][i] = in ? __ldcg(PI + (size_t)i * ncta + c) : 0x7fffffff;
        gv[j][i] = (in && GV) ? __ldcg(GV + (size_t)i * ncta + c) : -INFINITY;
        gi[j][i] = (in && GV) ? __ldcg(GI + (size_t)i * ncta + c) : 0x7fffffff;
      }
    }
#pragma unroll
    for (int j = 0; j < JP; ++j) lse_fold(ps[j], m, sum);
    fold_lists<KMAX, JP>(pv, pi, kb, L, I);
    if (GV) fold_lists<KMAX, JP>(gv, gi, kb, G, GI_);
  }
  const float lse = lse_finish(m, sum);
  emit_best<KMAX>(L, I, kb, lane, out_v, out_i);
  if (GV) emit_best<KMAX>(G, GI_, kb, lane, nullptr, out_g);
  return lse;
}

// One warp merges one of the lists of a node's ncta partials into its first
// kb entries.  out_v / out_i may be NULL when the values / tokens are not
// needed.
template <int KMAX>
__device__ __forceinline__ void merge_lists(const float* PV, const int32_t* PI, int ncta, int k,
                                            int kb, int lane, float* out_v, int32_t* out_i) {
  constexpr int JP = KMAX <= 4 ? 5 : 1;
  float L[KMAX];
  int32_t I[KMAX];
  list_init<KMAX>(L, I);
  for (int c0 = 0; c0 < ncta; c0 += 32 * JP) {
    float pv[JP][KMAX];
    int32_t pi[JP][KMAX];
#pragma unroll
    for (int j = 0; j < JP; ++j) {
      const int c = c0 + 32 * j + lane;
#pragma unroll
      for (int i = 0; i < KMAX; ++i) {
        const bool in = c < ncta && i < k;
        pv[j][i] = in ? __ldcg(PV + (size_t)i * ncta + c) : -INFINITY;
        pi[j][i] = in ? __ldcg(PI + (size_t)i * ncta + c) : 0x7fffffff;
      }
    }
    fold_lists<KMAX, JP>(pv, pi, kb, L, I);
  }
  emit_best<KMAX>(L, I, kb, lane, out_v, out_i);
}

// One warp merges the (max, sum exp) partials of a node into its log-sum-exp.
__device__ __forceinline__ float merge_lse(const float2* P, int ncta, int lane) {
  float m = -INFINITY, sv = 0.f;
  for (int c0 = 0; c0 < ncta; c0 += 32 * 5) {
    float2 ps[5];
#pragma unroll
    for (int j = 0; j < 5; ++j) {
      const int c = c0 + 32 * j + lane;
      ps[j] = c < ncta ? __ldcg(P + c) : make_float2(-INFINITY, 0.f);
    }
#pragma unroll
    for (int j = 0; j < 5; ++j) lse_fold(ps[j], m, sv);
  }
  return lse_finish(m, sv);
}

}  // namespace dt
